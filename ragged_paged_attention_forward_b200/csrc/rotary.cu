// The step's input pass with rotary position embedding: Q and K rows are rotated by their
// positions, Q goes to its output buffer and K, V into their cache slots.  Rotation rule
// ("[WebGPU] Optimized PagedAttention implementation (2/n)", commit "Phase 1b.2": position
// pos = past_b + s; interleaved or split pairing; dims >= rotary_dim copied unchanged), packed
// input layout (same page, packed-QKV commit: per token the columns [0, Hq D) hold Q, then
// Hkv D of K, then Hkv D of V), slot rule as in the KV scatter (commit "Phase 1b.1").
//
// B200 mapping: memory-bound row shuffling.  One warp per token: its sequence, position,
// page(s) and the cos/sin entries each lane needs are fetched once, then the token's rows
// (Hq query heads, Hkv key heads, Hkv value heads) go through two (D=128) or four (D=64) at
// a time, lane group g on row r0 + g.  Lane l of a row holds dims [8l, 8l + 8) (one 16-byte
// load); a split-mode pair (j, j + rd/2) spans lanes l and l + rd/16 of the row, whose values
// arrive by a shuffle, an interleaved pair sits inside one lane.
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

constexpr int kU = 4;  // row groups whose loads a warp keeps in flight

__global__ void __launch_bounds__(256, 4) rotary_write_kernel(RotaryLaunch p) {
  const int lane = threadIdx.x & 31;
  const int warps_per_block = blockDim.x >> 5;
  const int D = p.head_dim;
  const int lanes_row = D / 8;          // lanes holding one row (16 for D=128, 8 for D=64)
  const int rpi = 32 / lanes_row;       // rows per warp iteration
  const int sub = lane / lanes_row;     // which of those rows this lane works on
  const int l = lane - sub * lanes_row; // lane within the row: dims [8l, 8l + 8)
  const int d0 = l * 8;
  const int Hq = p.num_q_heads, Hkv = p.num_kv_heads;
  const int rows = Hq + 2 * Hkv;
  const bool packed = p.k == nullptr;
  const int rd = p.rotary_dim;
  const bool rot_any = p.cos != nullptr;
  const int half_lanes = rd / 16;       // split mode: lanes holding the first rd/2 dims
  const long nwarps = (long)gridDim.x * warps_per_block;
  // num_tokens is exact for host plans and a bound for device plans: the step's own count
  // is cu_seqlens_q[num_seqs]
  const int T = min(p.num_tokens, __ldg(p.cu_seqlens_q + p.num_seqs));
  for (long t = (long)blockIdx.x * warps_per_block + (threadIdx.x >> 5); t < T;
       t += nwarps) {
    // ---- per token: sequence, position, pages, the cos/sin entries of this lane's dims.
    // With at most 32 sequences the warp finds the sequence in one round of loads: lane i
    // reads cu_seqlens_q[i + 1] and seq_lens_k[i], and the sequence is the number of lanes
    // whose end is at or below t.
    int b, t0, q_len, pos;
    if (p.num_seqs <= 32) {
      const int cu_end = lane < p.num_seqs ? __ldg(p.cu_seqlens_q + lane + 1) : 0x7fffffff;
      const int kv_l = lane < p.num_seqs ? __ldg(p.seq_lens_k + lane) : 0;
      b = __popc(__ballot_sync(0xffffffffu, cu_end <= (int)t));
      const int end = __shfl_sync(0xffffffffu, cu_end, b & 31);
      const int prev_end = __shfl_sync(0xffffffffu, cu_end, (b + 31) & 31);
      t0 = b > 0 ? prev_end : 0;
      q_len = end - t0;
      pos = __shfl_sync(0xffffffffu, kv_l, b & 31) - q_len + ((int)t - t0);
    } else {
      b = seq_of_token(p.cu_seqlens_q, p.num_seqs, (int)t);
      t0 = __ldg(p.cu_seqlens_q + b);
      q_len = __ldg(p.cu_seqlens_q + b + 1) - t0;
      pos = __ldg(p.seq_lens_k + b) - q_len + ((int)t - t0);
    }
    const int blk = pos / p.page_size;
    const int slot = pos - blk * p.page_size;
    // page of KV head h (head-major: lane h holds it; sequence-major: one page for all)
    int page_l = -1;
    if (blk < p.max_blocks) {
      if (p.layout == 0)
        page_l = __ldg(p.block_table + (size_t)b * p.max_blocks + blk);
      else if (lane < Hkv)
        page_l = __ldg(p.block_table + ((size_t)b * Hkv + lane) * p.max_blocks + blk);
    }
    const bool rot_ok = rot_any && pos < p.max_pos;
    if (rot_any && !rot_ok && lane == 0) atomicOr(p.err, kErrBadPosition);
    uint32_t cs[4] = {0u, 0u, 0u, 0u}, sn[4] = {0u, 0u, 0u, 0u};
    if (rot_ok && d0 < rd) {
      const uint16_t* crow = p.cos + (size_t)pos * (rd / 2);
      const uint16_t* srow = p.sin + (size_t)pos * (rd / 2);
      if (p.interleaved) {  // pairs 4l .. 4l+3
        const uint2 c2 = __ldg(reinterpret_cast<const uint2*>(crow + d0 / 2));
        const uint2 s2 = __ldg(reinterpret_cast<const uint2*>(srow + d0 / 2));
        cs[0] = c2.x; cs[1] = c2.y; sn[0] = s2.x; sn[1] = s2.y;
      } else {              // pairs d0 .. d0+7 of the first or the second half
        const int j0 = l < half_lanes ? d0 : d0 - rd / 2;
        const uint4 c4 = __ldg(reinterpret_cast<const uint4*>(crow + j0));
        const uint4 s4 = __ldg(reinterpret_cast<const uint4*>(srow + j0));
        cs[0] = c4.x; cs[1] = c4.y; cs[2] = c4.z; cs[3] = c4.w;
        sn[0] = s4.x; sn[1] = s4.y; sn[2] = s4.z; sn[3] = s4.w;
      }
    }
    // ---- the token's rows, rpi at a time (Q heads, then K heads, then V heads), kU row
    // groups per round: all their loads are issued before any of them is used, so a warp
    // keeps kU * 512 bytes in flight
    for (int rb = 0; rb < rows; rb += kU * rpi) {
      uint4 xs[kU];
      int pages[kU];
      bool writes[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int r = rb + u * rpi + sub;
        const bool valid = r < rows;
        const int kind = r < Hq ? 0 : (r < Hq + Hkv ? 1 : 2);
        const int h = kind == 0 ? r : (kind == 1 ? r - Hq : r - Hq - Hkv);
        int page = page_l;
        if (p.layout != 0) {  // head-major: the page of KV head h (from lane h when Hkv <= 32)
          page = __shfl_sync(0xffffffffu, page_l, (valid && kind != 0 ? h : 0) & 31);
          if (Hkv > 32 && valid && kind != 0)
            page = blk < p.max_blocks
                       ? __ldg(p.block_table + ((size_t)b * Hkv + h) * p.max_blocks + blk)
                       : -1;
        }
        const bool rotate = rot_any && kind != 2;
        bool write = valid && !(rotate && !rot_ok);
        if (write && kind != 0 && (page < 0 || page >= p.num_pages)) {  // never write outside
          atomicOr(p.err, kErrBadIndex);
          write = false;
        }
        const uint16_t* src =
            packed ? p.q + ((size_t)t * rows + r) * D
                   : (kind == 0 ? p.q + ((size_t)t * Hq + h) * D
                                : (kind == 1 ? p.k : p.v) + ((size_t)t * Hkv + h) * D);
        // the load depends on nothing but the row, so it goes out before the metadata lands
        xs[u] = make_uint4(0u, 0u, 0u, 0u);
        if (valid) xs[u] = __ldg(reinterpret_cast<const uint4*>(src) + l);
        pages[u] = page;
        writes[u] = write;
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int r = rb + u * rpi + sub;
        const int kind = r < Hq ? 0 : (r < Hq + Hkv ? 1 : 2);
        const int h = kind == 0 ? r : (kind == 1 ? r - Hq : r - Hq - Hkv);
        const bool rotate = rot_any && kind != 2 && rot_ok && d0 < rd;
        uint32_t xw[4] = {xs[u].x, xs[u].y, xs[u].z, xs[u].w};
        if (rot_any) {  // warp-uniform: every lane takes part in the shuffles below
          if (p.interleaved) {
            if (rotate) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const float c = (k & 1) ? bf_hi(cs[k >> 1]) : bf_lo(cs[k >> 1]);
                const float s = (k & 1) ? bf_hi(sn[k >> 1]) : bf_lo(sn[k >> 1]);
                const float x1 = bf_lo(xw[k]), x2 = bf_hi(xw[k]);
                xw[k] = bf_pack(fmaf(x1, c, -x2 * s), fmaf(x1, s, x2 * c));
              }
            }
          } else {
            // pair j = (j, j + rd/2): lanes l and l + half_lanes of the same row swap values
            const int pl = l < half_lanes ? l + half_lanes : l - half_lanes;
            const int src_lane = (sub * lanes_row + (pl < lanes_row ? pl : l)) & 31;
            uint32_t pw[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) pw[k] = __shfl_sync(0xffffffffu, xw[k], src_lane);
            if (rotate) {
              const bool first = l < half_lanes;
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const float c0 = bf_lo(cs[k]), c1 = bf_hi(cs[k]);
                const float s0 = bf_lo(sn[k]), s1 = bf_hi(sn[k]);
                const float a0 = bf_lo(xw[k]), a1 = bf_hi(xw[k]);  // this lane's dims
                const float b0 = bf_lo(pw[k]), b1 = bf_hi(pw[k]);  // the partner dims
                // first half: own = x1 -> x1 c - x2 s; second half: own = x2 -> x1 s + x2 c
                const float r0v = first ? fmaf(a0, c0, -b0 * s0) : fmaf(b0, s0, a0 * c0);
                const float r1v = first ? fmaf(a1, c1, -b1 * s1) : fmaf(b1, s1, a1 * c1);
                xw[k] = bf_pack(r0v, r1v);
              }
            }
          }
        }
        if (writes[u]) {
          uint16_t* dst;
          if (kind == 0) {
            dst = p.q_out + ((size_t)t * Hq + h) * D;
          } else {
            uint16_t* pool = kind == 1 ? p.k_pool : p.v_pool;
            dst = pool + (p.layout == 0
                              ? (((size_t)pages[u] * p.page_size + slot) * Hkv + h) * D
                              : ((size_t)pages[u] * p.page_size + slot) * D);
          }
          reinterpret_cast<uint4*>(dst)[l] = make_uint4(xw[0], xw[1], xw[2], xw[3]);
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_rotary_write(const RotaryLaunch& p, cudaStream_t stream) {
  if (p.num_tokens <= 0) return cudaSuccess;
  const int threads = 256;
  long blocks = ((long)p.num_tokens + 7) / 8;  // one warp per token, 8 warps per block
  const long cap = (long)device_sm_count() * 64;
  if (blocks > cap) blocks = cap;
  rotary_write_kernel<<<(unsigned)blocks, threads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace rpa
