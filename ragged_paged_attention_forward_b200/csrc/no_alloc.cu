// rpa_forward_no_alloc: the fused step without a caller-supplied workspace.
//
// Some callers cannot allocate device memory on the path that runs the attention step: a
// host framework that owns every device byte (a serving engine whose allocator reserved the
// memory pool up front, or a plugin interface that hands the operator only its input and
// output tensors) has no way to give it a scratch buffer, and calling cudaMalloc there
// would stall the stream or fail.  For them the scratch this step needs -- the copied work
// lists and the split-KV decode partials merged afterwards -- lives in a fixed array that the
// library owns on every device that loads it.
#include <mutex>

#include "rpa.h"
#include "rpa_internal.h"

namespace {

constexpr size_t kStaticWorkspaceBytes = RPA_NO_ALLOC_WORKSPACE_BYTES;
constexpr int kMaxDevices = 64;

// The scratch itself.  Host code must not use this name as a device address: it is a
// host-side stand-in; the real address comes from cudaGetSymbolAddress on each device.
static __device__ __align__(256) uint8_t g_static_workspace[kStaticWorkspaceBytes];

void* g_workspace_addr[kMaxDevices] = {};
std::mutex g_workspace_mu;

// Device address of the array on the current device (looked up once per device).
rpa_status static_workspace(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    rpa::set_last_error("cudaGetDevice: %s", cudaGetErrorString(e));
    return RPA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    rpa::set_last_error("device %d is outside the %d devices this library tracks", dev,
                        kMaxDevices);
    return RPA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_workspace_mu);
  if (!g_workspace_addr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_static_workspace);
    if (e != cudaSuccess || !ptr) {
      rpa::set_last_error("cudaGetSymbolAddress(static workspace): %s", cudaGetErrorString(e));
      return RPA_ERR_CUDA;
    }
    g_workspace_addr[dev] = ptr;
  }
  *out = g_workspace_addr[dev];
  return RPA_OK;
}

}  // namespace

extern "C" rpa_status rpa_forward_no_alloc(rpa_plan_t plan, const void* q, const void* k_new,
                                           const void* v_new, void* k_pool, void* v_pool,
                                           const int32_t* block_table,
                                           const int32_t* cu_seqlens_q,
                                           const int32_t* seq_lens_k,
                                           const int32_t* group_table,
                                           const int32_t* group_count, float scale, void* out,
                                           float* lse, void* stream) {
  if (!plan) {
    rpa::set_last_error("plan must not be NULL");
    return RPA_ERR_INVALID_ARG;
  }
  rpa_plan_info info;
  rpa_status st = rpa_plan_get_info(plan, &info);
  if (st != RPA_OK) return st;
  if (info.workspace_bytes > kStaticWorkspaceBytes) {
    rpa::set_last_error(
        "this batch needs %zu bytes of scratch but the built-in workspace holds %zu bytes; "
        "call rpa_forward with a workspace of rpa_plan's size instead",
        info.workspace_bytes, kStaticWorkspaceBytes);
    return RPA_ERR_WORKSPACE_TOO_SMALL;
  }
  void* ws = nullptr;
  st = static_workspace(&ws);
  if (st != RPA_OK) return st;
  return rpa_forward(plan, q, k_new, v_new, k_pool, v_pool, block_table, cu_seqlens_q,
                     seq_lens_k, group_table, group_count, scale, out, lse, ws,
                     kStaticWorkspaceBytes, stream);
}

extern "C" size_t rpa_no_alloc_workspace_bytes(void) { return kStaticWorkspaceBytes; }
