// KV-cache scatter: the new tokens' K/V rows are copied, unchanged, into their page slots.
// Index rule ("[WebGPU] Optimized PagedAttention implementation (2/n)", squashed commit
// "Phase 1b.1", ScatterKVToPagedCacheProgram): token i of sequence b has absolute position
// pos = past_b + i (past_b = seq_lens_k[b] - q_len_b), page = block_table[b, pos / P],
// slot = pos % P.
//
// B200 mapping: one warp per token.  In the sequence-major pool a token's [Hkv, D] row of K
// (and of V) is one contiguous block at (page, slot) -- 2 KB for Llama-3-8B shapes -- so the
// warp moves it with 16-byte loads and stores; the head-major pool scatters one D-row per KV
// head.  The sequence of a token is found by binary search over cu_seqlens_q.
#include <cuda_fp16.h>

#include "ptx.cuh"
#include "rpa_internal.h"

namespace rpa {
namespace {

__device__ __forceinline__ int seq_of_token(const int32_t* __restrict__ cu, int B, int t) {
  int lo = 0, hi = B;  // answer in [0, B): cu[lo] <= t < cu[lo+1]
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (__ldg(cu + mid) <= t) lo = mid; else hi = mid;
  }
  return lo;
}

// e4m3 pools: one warp per token, one 16-byte output chunk (16 codes) per lane and step
__device__ void write_token_kv8(const WriteLaunch& p, int t, int b, int blk, int slot,
                                int lane) {
  const int chunks = p.head_dim / 16;                    // output chunks per D-row
  const int tok_chunks = p.num_kv_heads * chunks;
  for (int c = lane; c < tok_chunks; c += 32) {
    const int h = c / chunks;
    const int cc = c - h * chunks;
    const int page = p.layout == 0
                         ? __ldg(p.block_table + (size_t)b * p.max_blocks + blk)
                         : __ldg(p.block_table + ((size_t)b * p.num_kv_heads + h) * p.max_blocks +
                                 blk);
    if (page < 0 || page >= p.num_pages) {
      atomicOr(p.err, kErrBadIndex);
      continue;
    }
    const size_t row = p.layout == 0 ? ((size_t)page * p.page_size + slot) * p.num_kv_heads + h
                                     : (size_t)page * p.page_size + slot;
    const size_t src = ((size_t)t * p.num_kv_heads + h) * p.head_dim + cc * 16;
    const uint4* ks = reinterpret_cast<const uint4*>(p.k_new + src);
    const uint4* vs = reinterpret_cast<const uint4*>(p.v_new + src);
    uint8_t* kd = static_cast<uint8_t*>(p.k_pool) + row * p.head_dim + cc * 16;
    uint8_t* vd = static_cast<uint8_t*>(p.v_pool) + row * p.head_dim + cc * 16;
    *reinterpret_cast<uint4*>(kd) =
        e4m3_quantize16(__ldg(ks), __ldg(ks + 1), __ldg(p.k_scale + h));
    *reinterpret_cast<uint4*>(vd) =
        e4m3_quantize16(__ldg(vs), __ldg(vs + 1), __ldg(p.v_scale + h));
  }
}

__global__ void __launch_bounds__(256) write_kv_kernel(WriteLaunch p) {
  const int warps_per_block = blockDim.x >> 5;
  const int warp = blockIdx.x * warps_per_block + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * warps_per_block;
  const int row_chunks = p.head_dim / 8;                 // 16-byte chunks per D-row
  const int tok_chunks = p.num_kv_heads * row_chunks;   // chunks per token per K or V
  // device-planned steps: num_tokens is only a bound, the step's count is cu[num_seqs]
  const int T = p.tokens_on_device ? min(p.num_tokens, __ldg(p.cu_seqlens_q + p.num_seqs))
                                   : p.num_tokens;
  for (int t = warp; t < T; t += nwarps) {
    const int b = seq_of_token(p.cu_seqlens_q, p.num_seqs, t);
    const int t0 = __ldg(p.cu_seqlens_q + b);
    const int q_len = __ldg(p.cu_seqlens_q + b + 1) - t0;
    if (p.skip_rows_upto > 0 && q_len * p.group <= p.skip_rows_upto) continue;
    const int past = __ldg(p.seq_lens_k + b) - q_len;
    const int pos = past + (t - t0);
    if (p.below_box > 0 && pos >= (past + p.below_box - 1) / p.below_box * p.below_box) continue;
    const int blk = pos / p.page_size;
    const int slot = pos - blk * p.page_size;
    if (pos < 0 || blk >= p.max_blocks) {  // a device-planned step past its limits
      if (lane == 0) atomicOr(p.err, kErrLimits);
      continue;
    }
    if (p.kv8) {
      write_token_kv8(p, t, b, blk, slot, lane);
      continue;
    }
    const uint4* ksrc = reinterpret_cast<const uint4*>(p.k_new + (size_t)t * tok_chunks * 8);
    const uint4* vsrc = reinterpret_cast<const uint4*>(p.v_new + (size_t)t * tok_chunks * 8);
    if (p.layout == 0) {
      const int page = __ldg(p.block_table + (size_t)b * p.max_blocks + blk);
      if (page < 0 || page >= p.num_pages) {  // never write outside the pool
        if (lane == 0) atomicOr(p.err, kErrBadIndex);
        continue;
      }
      const size_t base = ((size_t)page * p.page_size + slot) * tok_chunks;
      uint4* kdst = reinterpret_cast<uint4*>(p.k_pool) + base;
      uint4* vdst = reinterpret_cast<uint4*>(p.v_pool) + base;
      for (int c = lane; c < tok_chunks; c += 32) {
        kdst[c] = __ldg(ksrc + c);
        vdst[c] = __ldg(vsrc + c);
      }
    } else {
      for (int c = lane; c < tok_chunks; c += 32) {
        const int h = c / row_chunks;
        const int cc = c - h * row_chunks;
        const int page =
            __ldg(p.block_table + ((size_t)b * p.num_kv_heads + h) * p.max_blocks + blk);
        if (page < 0 || page >= p.num_pages) {
          atomicOr(p.err, kErrBadIndex);
          continue;
        }
        const size_t base = ((size_t)page * p.page_size + slot) * row_chunks + cc;
        reinterpret_cast<uint4*>(p.k_pool)[base] = __ldg(ksrc + c);
        reinterpret_cast<uint4*>(p.v_pool)[base] = __ldg(vsrc + c);
      }
    }
  }
}

}  // namespace

cudaError_t launch_write_kv(const WriteLaunch& p, cudaStream_t stream) {
  if (p.num_tokens <= 0) return cudaSuccess;
  const int threads = 256;
  const int warps = threads / 32;
  int blocks = (p.num_tokens + warps - 1) / warps;
  const int cap = device_sm_count() * 8;
  if (blocks > cap) blocks = cap;
  write_kv_kernel<<<blocks, threads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace rpa
