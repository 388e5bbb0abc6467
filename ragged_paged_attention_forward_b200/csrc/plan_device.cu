// The planner on the device: the same work lists rpa_plan builds on the host (decode items
// per key split, merge rows, 128-query prefill tiles; "Ragged Paged Attention ..." Key ideas,
// the per-sequence slicing of a ragged batch), built from the step's device lengths so that
// a step needs no host arrays and can be captured in a CUDA graph.
//
// One CTA of 1024 threads walks the sequences 1024 at a time: each thread sizes its
// sequence's share of every list, a block-wide exclusive scan (warp shuffles, then the 32
// warp totals) turns the sizes into offsets, and each thread writes its entries.  The lists
// keep sequence order (the host planner sorts them heaviest first); a sequence's prefill
// tiles go last tile first, the causal tile with the most keys leading.  Counts land in
// counts[0..2]; a step beyond the plan's limits raises kErrLimits and computes nothing.
#include "rpa_internal.h"

namespace rpa {
namespace {

constexpr int kPlanThreads = 1024;

// exclusive prefix sums over the block of four values per thread; returns the block totals
__device__ __forceinline__ void block_scan4(int (&v)[4], int (&total)[4],
                                            int (*warp_sums)[4]) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  int incl[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    incl[k] = v[k];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl[k], off);
      if (lane >= off) incl[k] += y;
    }
  }
  if (lane == 31) {
#pragma unroll
    for (int k = 0; k < 4; ++k) warp_sums[warp][k] = incl[k];
  }
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      int x = warp_sums[lane][k];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
      }
      warp_sums[lane][k] = x;  // inclusive over warps
    }
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int before = warp > 0 ? warp_sums[warp - 1][k] : 0;
    total[k] = warp_sums[31][k];
    v[k] = before + incl[k] - v[k];
  }
  __syncthreads();  // warp_sums is reused by the next 1024 sequences
}

__global__ void __launch_bounds__(kPlanThreads) plan_device_kernel(PlanDeviceLaunch p) {
  __shared__ int warp_sums[32][4];
  const int G = p.num_q_heads / p.num_kv_heads;
  int base[4] = {0, 0, 0, 0};  // items, partial slots, merge rows, tiles placed so far
  bool over = false;
  for (int b0 = 0; b0 < p.num_seqs; b0 += kPlanThreads) {
    const int b = b0 + threadIdx.x;
    int t0 = 0, q_len = 0, kv = 0;
    int n[4] = {0, 0, 0, 0};  // items, slots, merge rows, tiles of this sequence
    bool dec = false;
    if (b < p.num_seqs) {
      t0 = __ldg(p.cu_seqlens_q + b);
      q_len = __ldg(p.cu_seqlens_q + b + 1) - t0;
      kv = __ldg(p.seq_lens_k + b);
      const bool ok = t0 >= 0 && q_len >= 0 && q_len <= kv && kv <= p.max_kv_len &&
                      t0 + q_len <= p.max_tokens;
      if (!ok) {
        atomicOr(p.err, kErrLimits);
        q_len = 0;
      }
      if (q_len > 0) {
        dec = q_len * G <= p.decode_rows;
        if (dec) {
          n[0] = (kv + p.split_keys - 1) / p.split_keys;
          if (n[0] > 1) {
            n[1] = n[0];
            n[2] = q_len;
          }
        } else {
          n[3] = (q_len + kPrefillTileRows - 1) / kPrefillTileRows;
        }
      }
    }
    int off[4] = {n[0], n[1], n[2], n[3]};
    int total[4];
    block_scan4(off, total, warp_sums);
#pragma unroll
    for (int k = 0; k < 4; ++k) off[k] += base[k];
    const bool fits = off[0] + n[0] <= p.cap_items && off[1] + n[1] <= p.cap_items &&
                      off[2] + n[2] <= p.cap_rows && off[3] + n[3] <= p.cap_tiles;
    if (!fits) over = true;
    if (b < p.num_seqs && fits) {
      for (int sp = 0; sp < n[0]; ++sp) {
        DecodeItem it;
        it.seq = b;
        it.t0 = t0;
        it.q_len = q_len;
        it.kv_len = kv;
        it.k_begin = sp * p.split_keys;
        it.k_end = min(kv, (sp + 1) * p.split_keys);
        it.part_slot = n[1] > 0 ? off[1] + sp : -1;
        it.pad = 0;
        p.items[off[0] + sp] = it;
      }
      for (int i = 0; i < n[2]; ++i) {
        MergeRow mr;
        mr.token = t0 + i;
        mr.local = i;
        mr.first_slot = off[1];
        mr.nsplit = n[0];
        p.rows[off[2] + i] = mr;
      }
      for (int k = 0; k < n[3]; ++k) {
        PrefillTile tl;
        tl.seq = b;
        tl.t0 = t0;
        tl.q_len = q_len;
        tl.kv_len = kv;
        tl.q_start = (n[3] - 1 - k) * kPrefillTileRows;
        tl.pad[0] = tl.pad[1] = tl.pad[2] = 0;
        p.tiles[off[3] + k] = tl;
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) base[k] += total[k];
  }
  // a step that does not fit computes nothing (its lists could have holes) and says so
  const bool any_over = __syncthreads_or(over);
  if (threadIdx.x == 0) {
    if (any_over) atomicOr(p.err, kErrLimits);
    p.counts[0] = any_over ? 0 : base[0];
    p.counts[1] = any_over ? 0 : base[2];
    p.counts[2] = any_over ? 0 : base[3];
  }
}

}  // namespace

cudaError_t launch_plan_device(const PlanDeviceLaunch& p, cudaStream_t stream) {
  plan_device_kernel<<<1, kPlanThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace rpa
