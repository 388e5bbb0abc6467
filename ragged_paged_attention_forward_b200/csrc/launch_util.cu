// Host-side launch helpers: TMA tensor maps (encoded through the driver entry point, so the
// library needs no link-time libcuda), per-device kernel attributes, the device error word.
#include <cudaTypedefs.h>

#include <mutex>
#include <vector>

#include "rpa_internal.h"

namespace rpa {

namespace {

// The library's device error word.  Kernels OR a DeviceErrorCode into it when a bounded wait
// runs out or an index is out of range; rpa_device_error() reads and clears it.
__device__ int g_device_error = 0;

constexpr int kMaxDevices = 64;

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

int current_device() {
  int dev = 0;
  cudaGetDevice(&dev);
  return dev;
}

}  // namespace

cudaError_t encode_kv_map(CUtensorMap* map, const void* pool, const PagedKV& kv, int head_dim,
                          int box_keys) {
  auto enc = tensor_map_encoder();
  if (!enc) {
    set_last_error("cuTensorMapEncodeTiled is not available from the driver");
    return cudaErrorNotSupported;
  }
  const uint64_t heads = kv.layout == 0 ? (uint64_t)kv.num_kv_heads : 1ull;
  // bf16 pools: boxes of 64 elements (128 bytes); e4m3 pools: 128 one-byte codes
  const uint64_t eb = kv.kv8 ? 1 : 2;
  cuuint64_t dims[4] = {(cuuint64_t)head_dim, heads, (cuuint64_t)kv.page_size,
                        (cuuint64_t)kv.num_pages};
  cuuint64_t strides[3] = {(cuuint64_t)head_dim * eb, (cuuint64_t)heads * head_dim * eb,
                           (cuuint64_t)kv.page_size * heads * head_dim * eb};
  const int rows = kv.page_size < box_keys ? kv.page_size : box_keys;
  cuuint32_t box[4] = {(cuuint32_t)(128 / eb), 1, (cuuint32_t)rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, kv.kv8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                   4, const_cast<void*>(pool), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B,
                   // a box row is 128 bytes; bf16 rows come in two halves (256 bytes
                   // together), e4m3 rows are one 128-byte run at a stride of Hkv*D bytes
                   kv.kv8 ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B : CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_last_error("cuTensorMapEncodeTiled(kv) failed with CUresult %d", (int)r);
    return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

cudaError_t encode_q_map(CUtensorMap* map, const void* q, int num_tokens, int num_q_heads,
                         int head_dim, int box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) {
    set_last_error("cuTensorMapEncodeTiled is not available from the driver");
    return cudaErrorNotSupported;
  }
  cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)num_q_heads, (cuuint64_t)num_tokens};
  cuuint64_t strides[2] = {(cuuint64_t)head_dim * 2, (cuuint64_t)num_q_heads * head_dim * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_last_error("cuTensorMapEncodeTiled(q) failed with CUresult %d", (int)r);
    return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

cudaError_t ensure_smem_attr(const void* kernel, int bytes) {
  // (kernel, device) pairs already raised; a handful of kernels, so a small table suffices
  struct Entry {
    const void* kernel;
    int device;
    int bytes;
  };
  static Entry table[256];
  static int used = 0;
  static std::mutex mu;
  const int dev = current_device();
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (table[i].kernel == kernel && table[i].device == dev && table[i].bytes >= bytes)
      return cudaSuccess;
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  if (used < 256) table[used++] = Entry{kernel, dev, bytes};
  return cudaSuccess;
}

cudaError_t side_stream(cudaStream_t caller, cudaStream_t* stream) {
  // one side stream per (device, caller stream), so that callers on different streams do
  // not serialise their tensor-core work on a shared one; past kMaxSideStreams caller streams
  // on a device, later callers share the existing side streams (correct, less concurrent)
  constexpr size_t kMaxSideStreams = 64;
  struct Entry {
    cudaStream_t caller;
    cudaStream_t side;
  };
  static std::vector<Entry> table[kMaxDevices];
  static std::mutex mu;
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  std::vector<Entry>& t = table[dev];
  for (const Entry& e : t)
    if (e.caller == caller) {
      *stream = e.side;
      return cudaSuccess;
    }
  if (t.size() >= kMaxSideStreams) {
    *stream = t[(reinterpret_cast<uintptr_t>(caller) >> 4) % t.size()].side;
    return cudaSuccess;
  }
  cudaStream_t side = nullptr;
  cudaError_t e = cudaStreamCreateWithFlags(&side, cudaStreamNonBlocking);
  if (e != cudaSuccess) return e;
  t.push_back(Entry{caller, side});
  *stream = side;
  return cudaSuccess;
}

int device_sm_count() {
  static int counts[kMaxDevices] = {0};
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 148;
  if (counts[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    counts[dev] = n;
  }
  return counts[dev];
}

cudaError_t device_error_word(int** ptr) {
  static int* addrs[kMaxDevices] = {nullptr};
  static std::mutex mu;
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addrs[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_device_error);
    if (e != cudaSuccess) return e;
    addrs[dev] = static_cast<int*>(p);
  }
  *ptr = addrs[dev];
  return cudaSuccess;
}

}  // namespace rpa
