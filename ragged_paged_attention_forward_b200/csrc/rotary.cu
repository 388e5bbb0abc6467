// The step's input pass with rotary position embedding: Q and K rows are rotated by their
// positions, Q goes to its output buffer and K, V into their cache slots.  Rotation rule
// ("[WebGPU] Optimized PagedAttention implementation (2/n)", commit "Phase 1b.2": position
// pos = past_b + s; interleaved or split pairing; dims >= rotary_dim copied unchanged), packed
// input layout (same page, packed-QKV commit: per token the columns [0, Hq D) hold Q, then
// Hkv D of K, then Hkv D of V), slot rule as in the KV scatter (commit "Phase 1b.1").
//
// B200 mapping: memory-bound row shuffling.  One warp per (token, row) with rows = Hq query
// heads, then Hkv key heads, then Hkv value heads.  Lane l holds dims [8l, 8l + 8) of the row
// (one 16-byte load); a split-mode pair (j, j + rd/2) spans lanes l and l + rd/16, whose
// values arrive by a shuffle, an interleaved pair sits inside one lane.  The cos/sin rows of
// the position are read with one 16-byte load per lane (8 entries, or 4 pairs).
#include <cuda_bf16.h>

#include "rpa_internal.h"

namespace rpa {
namespace {

__device__ __forceinline__ int seq_of_token(const int32_t* __restrict__ cu, int B, int t) {
  int lo = 0, hi = B;  // answer in [0, B): cu[lo] <= t < cu[lo+1]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(cu + mid) <= t) lo = mid; else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ uint32_t bf_pack(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__global__ void __launch_bounds__(256) rotary_write_kernel(RotaryLaunch p) {
  const int lane = threadIdx.x & 31;
  const int warps_per_block = blockDim.x >> 5;
  const int D = p.head_dim;
  const int lanes_row = D / 8;                      // lanes holding a row (16 or 8)
  const int rows = p.num_q_heads + 2 * p.num_kv_heads;
  const long total = (long)p.num_tokens * rows;
  const long nwarps = (long)gridDim.x * warps_per_block;
  const bool packed = p.k == nullptr;
  const int rd = p.rotary_dim;
  for (long w = (long)blockIdx.x * warps_per_block + (threadIdx.x >> 5); w < total;
       w += nwarps) {
    const int t = (int)(w / rows);
    const int r = (int)(w - (long)t * rows);      // row within the token: Q heads, K, V
    const int kind = r < p.num_q_heads ? 0 : (r < p.num_q_heads + p.num_kv_heads ? 1 : 2);
    const int h = kind == 0 ? r : (kind == 1 ? r - p.num_q_heads
                                             : r - p.num_q_heads - p.num_kv_heads);
    const int b = seq_of_token(p.cu_seqlens_q, p.num_seqs, t);
    const int t0 = __ldg(p.cu_seqlens_q + b);
    const int q_len = __ldg(p.cu_seqlens_q + b + 1) - t0;
    const int pos = __ldg(p.seq_lens_k + b) - q_len + (t - t0);
    // source row
    const uint16_t* src;
    if (packed) {
      src = p.q + (size_t)t * rows * D + (size_t)r * D;
    } else {
      src = kind == 0 ? p.q + ((size_t)t * p.num_q_heads + h) * D
                      : (kind == 1 ? p.k : p.v) + ((size_t)t * p.num_kv_heads + h) * D;
    }
    // destination row
    uint16_t* dst = nullptr;
    if (kind == 0) {
      dst = p.q_out + ((size_t)t * p.num_q_heads + h) * D;
    } else {
      const int blk = pos / p.page_size;
      const int slot = pos - blk * p.page_size;
      const int page =
          blk < p.max_blocks
              ? __ldg(p.block_table + (p.layout == 0
                                           ? (size_t)b * p.max_blocks + blk
                                           : ((size_t)b * p.num_kv_heads + h) * p.max_blocks +
                                                 blk))
              : -1;
      if (page < 0 || page >= p.num_pages) {  // never write outside the pool
        if (lane == 0) atomicOr(p.err, kErrBadIndex);
        continue;
      }
      uint16_t* pool = kind == 1 ? p.k_pool : p.v_pool;
      dst = pool + (p.layout == 0 ? (((size_t)page * p.page_size + slot) * p.num_kv_heads + h) * D
                                  : ((size_t)page * p.page_size + slot) * D);
    }
    const bool rotate = p.cos != nullptr && kind != 2;
    if (rotate && pos >= p.max_pos) {
      if (lane == 0) atomicOr(p.err, kErrBadPosition);
      continue;
    }
    uint4 x = make_uint4(0u, 0u, 0u, 0u);
    if (lane < lanes_row) x = __ldg(reinterpret_cast<const uint4*>(src) + lane);
    if (rotate) {
      const int d0 = lane * 8;  // first dim of this lane
      uint32_t xw[4] = {x.x, x.y, x.z, x.w};
      if (p.interleaved) {
        // pairs (2j, 2j+1) inside the lane: pairs 4l .. 4l+3
        if (lane < lanes_row && d0 < rd) {
          const uint2 cw = __ldg(reinterpret_cast<const uint2*>(p.cos + (size_t)pos * (rd / 2) +
                                                                 d0 / 2));
          const uint2 sw = __ldg(reinterpret_cast<const uint2*>(p.sin + (size_t)pos * (rd / 2) +
                                                                 d0 / 2));
          const uint32_t cs[2] = {cw.x, cw.y}, sn[2] = {sw.x, sw.y};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float c = (k & 1) ? bf_hi(cs[k >> 1]) : bf_lo(cs[k >> 1]);
            const float s = (k & 1) ? bf_hi(sn[k >> 1]) : bf_lo(sn[k >> 1]);
            const float x1 = bf_lo(xw[k]), x2 = bf_hi(xw[k]);
            xw[k] = bf_pack(fmaf(x1, c, -x2 * s), fmaf(x1, s, x2 * c));
          }
        }
      } else {
        // pair j = (j, j + rd/2): the lane with the first half fetches its partner's dims
        const int half_lanes = rd / 16;  // lanes holding the first rd/2 dims
        uint32_t pw[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          // first-half lanes read lane + half_lanes; second-half lanes read lane - half_lanes
          const int src_lane = lane < half_lanes ? lane + half_lanes : lane - half_lanes;
          pw[k] = __shfl_sync(0xffffffffu, xw[k], src_lane & 31);
        }
        if (lane < lanes_row && d0 < rd) {
          const bool first = lane < half_lanes;
          const int j0 = first ? d0 : d0 - rd / 2;  // pair index of this lane's first dim
          const uint4 cw = __ldg(reinterpret_cast<const uint4*>(p.cos + (size_t)pos * (rd / 2) +
                                                                 j0));
          const uint4 sw = __ldg(reinterpret_cast<const uint4*>(p.sin + (size_t)pos * (rd / 2) +
                                                                 j0));
          const uint32_t cs[4] = {cw.x, cw.y, cw.z, cw.w}, sn[4] = {sw.x, sw.y, sw.z, sw.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float c0 = bf_lo(cs[k]), c1 = bf_hi(cs[k]);
            const float s0 = bf_lo(sn[k]), s1 = bf_hi(sn[k]);
            const float a0 = bf_lo(xw[k]), a1 = bf_hi(xw[k]);  // this lane's dims
            const float b0 = bf_lo(pw[k]), b1 = bf_hi(pw[k]);  // the partner dims
            // first half: x1 = own, x2 = partner -> x1 c - x2 s
            // second half: x2 = own, x1 = partner -> x1 s + x2 c
            const float r0 = first ? fmaf(a0, c0, -b0 * s0) : fmaf(b0, s0, a0 * c0);
            const float r1 = first ? fmaf(a1, c1, -b1 * s1) : fmaf(b1, s1, a1 * c1);
            xw[k] = bf_pack(r0, r1);
          }
        }
      }
      x = make_uint4(xw[0], xw[1], xw[2], xw[3]);
    }
    if (lane < lanes_row) reinterpret_cast<uint4*>(dst)[lane] = x;
  }
}

}  // namespace

cudaError_t launch_rotary_write(const RotaryLaunch& p, cudaStream_t stream) {
  if (p.num_tokens <= 0) return cudaSuccess;
  const int threads = 256;
  const long rows = (long)p.num_tokens * (p.num_q_heads + 2 * p.num_kv_heads);
  long blocks = (rows + 7) / 8;
  const long cap = (long)device_sm_count() * 16;
  if (blocks > cap) blocks = cap;
  rotary_write_kernel<<<(unsigned)blocks, threads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace rpa
