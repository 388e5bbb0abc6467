// Block-union KV selection ("CompactAttention: Accelerating Chunked Prefill with Block-Union
// KV Selection", Core claim and Fig. 3): a per-head 2-D block mask [B, Hq, nqb, nkb] becomes,
// for every (sequence, KV group), the ascending list of KV blocks that some query head of
// the group selects in some query block.
//
// One CTA per (sequence, KV group).  Each thread ORs the G x nqb mask bytes of one KV block
// (consecutive threads read consecutive bytes), the block computes an exclusive prefix sum of
// the selection flags with warp ballots, and the selected block indices are stored in order;
// the rest of the row is filled with -1.  The result is deterministic and bit-exact.
#include "rpa_internal.h"

namespace rpa {
namespace {

constexpr int kThreads = 512;

__global__ void __launch_bounds__(kThreads) group_tables_kernel(const uint8_t* __restrict__ mask,
                                                                int Hq, int Hkv, int nqb, int nkb,
                                                                int32_t* __restrict__ table,
                                                                int32_t* __restrict__ count) {
  __shared__ int warp_tot[kThreads / 32];
  __shared__ int base_sh;
  const int b = blockIdx.x / Hkv;
  const int g = blockIdx.x - b * Hkv;
  const int G = Hq / Hkv;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const size_t head_stride = (size_t)nqb * nkb;
  const uint8_t* m0 = mask + ((size_t)b * Hq + (size_t)g * G) * head_stride;
  int32_t* row = table + ((size_t)b * Hkv + g) * nkb;
  if (threadIdx.x == 0) base_sh = 0;
  __syncthreads();
  for (int start = 0; start < nkb; start += kThreads) {
    const int kb = start + threadIdx.x;
    int sel = 0;
    if (kb < nkb) {
      for (int hh = 0; hh < G && !sel; ++hh)
        for (int qb = 0; qb < nqb; ++qb)
          if (__ldg(m0 + hh * head_stride + (size_t)qb * nkb + kb)) {
            sel = 1;
            break;
          }
    }
    const unsigned ballot = __ballot_sync(0xffffffffu, sel);
    const int in_warp = __popc(ballot & ((1u << lane) - 1u));
    if (lane == 0) warp_tot[warp] = __popc(ballot);
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < kThreads / 32; ++w) {
      const int c = warp_tot[w];
      if (w < warp) before += c;
      total += c;
    }
    const int base = base_sh;
    if (sel) row[base + before + in_warp] = kb;
    __syncthreads();
    if (threadIdx.x == 0) base_sh = base + total;
    __syncthreads();
  }
  const int n = base_sh;
  for (int i = n + threadIdx.x; i < nkb; i += kThreads) row[i] = -1;
  if (threadIdx.x == 0) count[(size_t)b * Hkv + g] = n;
}

}  // namespace

cudaError_t launch_group_tables(const uint8_t* mask, int B, int Hq, int Hkv, int nqb, int nkb,
                                int32_t* table, int32_t* count, cudaStream_t stream) {
  if (B <= 0 || Hkv <= 0) return cudaSuccess;
  group_tables_kernel<<<B * Hkv, kThreads, 0, stream>>>(mask, Hq, Hkv, nqb, nkb, table, count);
  return cudaGetLastError();
}

}  // namespace rpa
