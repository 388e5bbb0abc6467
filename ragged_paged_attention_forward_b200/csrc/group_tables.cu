// Block-union KV selection ("CompactAttention: Accelerating Chunked Prefill with Block-Union
// KV Selection", Core claim and Fig. 3): a per-head 2-D block mask [B, Hq, nqb, nkb] becomes,
// for every (sequence, KV group), the ascending list of KV blocks that some query head of
// the group selects in some query block.
//
// One CTA per (sequence, KV group); the selected block indices are stored in ascending order
// and the rest of the row is filled with -1.  Deterministic and bit-exact.  Byte-wise path:
// each thread ORs the G x nqb mask bytes of one KV block and the block compacts the flags with
// warp ballots.
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

// Vector path (nkb a multiple of 16, mask 16-byte aligned): 1024 threads = 8 row groups x 128
// threads; a thread ORs 16 consecutive KV blocks (one 16-byte load per mask row) over its row
// group's share of the G*nqb rows, the 8 partial ORs are combined in shared memory, and the
// first 128 threads turn the 16 bytes into 16 selection bits and compact them in order.
constexpr int kVecThreads = 1024;
constexpr int kVecGroups = 8;
constexpr int kVecLanes = kVecThreads / kVecGroups;  // 128 threads -> 2048 blocks per chunk
constexpr int kVecBlocks = kVecLanes * 16;

__global__ void __launch_bounds__(kVecThreads) group_tables_vec_kernel(
    const uint8_t* __restrict__ mask, int Hq, int Hkv, int nqb, int nkb,
    int32_t* __restrict__ table, int32_t* __restrict__ count) {
  __shared__ uint4 part[kVecGroups][kVecLanes];
  __shared__ int warp_tot[kVecLanes / 32];
  __shared__ int base_sh;
  const int b = blockIdx.x / Hkv;
  const int g = blockIdx.x - b * Hkv;
  const int G = Hq / Hkv;
  const int rows = G * nqb;  // rows of the group: (head, q-block), each nkb bytes
  const int grp = threadIdx.x / kVecLanes;
  const int lt = threadIdx.x - grp * kVecLanes;
  const uint8_t* m0 = mask + ((size_t)b * Hq + (size_t)g * G) * nqb * nkb;
  int32_t* row_out = table + ((size_t)b * Hkv + g) * nkb;
  if (threadIdx.x == 0) base_sh = 0;
  __syncthreads();
  for (int kb0 = 0; kb0 < nkb; kb0 += kVecBlocks) {
    const int kb = kb0 + lt * 16;
    uint4 acc = make_uint4(0u, 0u, 0u, 0u);
    if (kb < nkb) {
#pragma unroll 4
      for (int r = grp; r < rows; r += kVecGroups) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(m0 + (size_t)r * nkb + kb));
        acc.x |= v.x;
        acc.y |= v.y;
        acc.z |= v.z;
        acc.w |= v.w;
      }
    }
    part[grp][lt] = acc;
    __syncthreads();
    if (grp == 0) {
      uint4 o = part[0][lt];
#pragma unroll
      for (int k = 1; k < kVecGroups; ++k) {
        o.x |= part[k][lt].x;
        o.y |= part[k][lt].y;
        o.z |= part[k][lt].z;
        o.w |= part[k][lt].w;
      }
      const uint32_t w[4] = {o.x, o.y, o.z, o.w};
      uint32_t sel = 0;  // bit i: block kb + i selected
#pragma unroll
      for (int i = 0; i < 16; ++i) sel |= (((w[i >> 2] >> ((i & 3) * 8)) & 0xffu) ? 1u : 0u) << i;
      if (kb >= nkb) sel = 0;
      const int n = __popc(sel);
      // exclusive scan of n over the 128 threads (4 warps), in kb order
      const int lane = lt & 31, wp = lt >> 5;
      int incl = n;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      if (lane == 31) warp_tot[wp] = incl;
      asm volatile("bar.sync 1, %0;" ::"n"(kVecLanes));
      int before = 0, total = 0;
#pragma unroll
      for (int k = 0; k < kVecLanes / 32; ++k) {
        if (k < wp) before += warp_tot[k];
        total += warp_tot[k];
      }
      int pos = base_sh + before + incl - n;
      for (uint32_t s2 = sel; s2; s2 &= s2 - 1) row_out[pos++] = kb + __ffs(s2) - 1;
      asm volatile("bar.sync 1, %0;" ::"n"(kVecLanes));
      if (lt == 0) base_sh += total;
    }
    __syncthreads();
  }
  const int n = base_sh;
  for (int i = n + threadIdx.x; i < nkb; i += kVecThreads) row_out[i] = -1;
  if (threadIdx.x == 0) count[(size_t)b * Hkv + g] = n;
}

// Per-(query tile, query head) tables: the execution of a block-sparse kernel that works per
// query block and head (the comparison of CompactAttention's Fig. 7c, execution-only ablation
// with the same mask).  Row (b, hq, tile) lists, in ascending order, the KV blocks that head hq
// selects in any query block of the 128-row query tile; the rest of the row is -1.  One CTA
// per row; the same ballot compaction as group_tables_kernel.
__global__ void __launch_bounds__(kThreads) qtile_tables_kernel(
    const uint8_t* __restrict__ mask, int Hq, int nqb, int nkb, int qb_per_tile, int ntiles,
    int32_t* __restrict__ table, int32_t* __restrict__ count) {
  __shared__ int warp_tot[kThreads / 32];
  __shared__ int base_sh;
  const int tile = blockIdx.x % ntiles;
  const int hq = (blockIdx.x / ntiles) % Hq;
  const int b = blockIdx.x / (ntiles * Hq);
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const uint8_t* m0 = mask + ((size_t)b * Hq + hq) * nqb * nkb;
  const int qb0 = tile * qb_per_tile;
  const int qb1 = min(nqb, qb0 + qb_per_tile);
  int32_t* row = table + (((size_t)b * Hq + hq) * ntiles + tile) * nkb;
  if (threadIdx.x == 0) base_sh = 0;
  __syncthreads();
  for (int start = 0; start < nkb; start += kThreads) {
    const int kb = start + threadIdx.x;
    int sel = 0;
    if (kb < nkb)
      for (int qb = qb0; qb < qb1 && !sel; ++qb) sel = __ldg(m0 + (size_t)qb * nkb + kb) != 0;
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
  if (threadIdx.x == 0) count[((size_t)b * Hq + hq) * ntiles + tile] = n;
}

}  // namespace

cudaError_t launch_qtile_tables(const uint8_t* mask, int B, int Hq, int nqb, int nkb,
                                int qb_per_tile, int ntiles, int32_t* table, int32_t* count,
                                cudaStream_t stream) {
  if (B <= 0 || ntiles <= 0) return cudaSuccess;
  qtile_tables_kernel<<<B * Hq * ntiles, kThreads, 0, stream>>>(mask, Hq, nqb, nkb, qb_per_tile,
                                                                ntiles, table, count);
  return cudaGetLastError();
}

cudaError_t launch_group_tables(const uint8_t* mask, int B, int Hq, int Hkv, int nqb, int nkb,
                                int32_t* table, int32_t* count, cudaStream_t stream) {
  if (B <= 0 || Hkv <= 0) return cudaSuccess;
  if (nkb % 16 == 0 && (reinterpret_cast<uintptr_t>(mask) & 15u) == 0)
    group_tables_vec_kernel<<<B * Hkv, kVecThreads, 0, stream>>>(mask, Hq, Hkv, nqb, nkb, table,
                                                                 count);
  else
    group_tables_kernel<<<B * Hkv, kThreads, 0, stream>>>(mask, Hq, Hkv, nqb, nkb, table,
                                                          count);
  return cudaGetLastError();
}

}  // namespace rpa
