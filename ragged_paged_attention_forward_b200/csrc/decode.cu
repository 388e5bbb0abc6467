// Split-KV decode over the paged cache, and the log-sum-exp merge of the splits.
//
// What it computes: for every (sequence, KV head, key split) the partial softmax attention of
// the sequence's short query (q_len * G <= 32 rows: every query head of the KV group for
// every query token) over keys [k_begin, k_end), read in place through the block table.  This
// is the split-reduce decode of "[WebGPU] Optimized PagedAttention implementation (2/n)"
// ("What's shipped": FlashAttentionPagedDecodeQKV + FlashAttentionPagedDecodeVxReduce,
// selected for max_seqlen_q < 32) and the decode specialisation of "Ragged Paged Attention:
// A High-Performance and Flexible LLM Inference Kernel for TPU" (Key ideas).
//
// B200 design:
//  * one producer warp streams the split's pages with TMA (one block-table lookup per page,
//    not per slot): boxes of [min(P, 64) slots x 64 dims] per page and half-row, 128-byte
//    swizzled, into a 3-4 stage ring of 64-key stages completed on mbarriers;
//  * four consumer warps each own 16 keys of a stage.  S^T = K Q^T runs on the tensor cores
//    (mma.sync m16n8k16, keys in M, the G heads x q tokens of the group in N), the online
//    softmax works per query column with three shuffles, P^T is turned into the B operand by
//    movmatrix, and O^T += V^T P^T runs on the tensor cores again; K and V are read from HBM
//    exactly once per KV group;
//  * the four warps' states are combined in shared memory; a sequence with one split writes
//    the final bf16 output, otherwise the split's normalised output and log2-domain LSE go to
//    the workspace for the merge kernel.
//  Key slots past k_end (the tail of the last page, possibly NaN) are masked in S and their V
//  rows are zeroed in shared memory before the P.V product.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "ptx.cuh"
#include "rpa_internal.h"

namespace rpa {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxItemPages = kMaxSplitKeys / 16 + 1;

template <int D, bool KV8, int NT>
struct DecodeGeom {
  // stage rows are stored in 128-byte halves: 64 bf16 elements, or all 128 e4m3 codes
  static constexpr int kHalves = KV8 ? 1 : D / 64;
  static constexpr int kStageKeys = kDecodeStageKeys;                 // 64
  static constexpr int kHalfBytes = kStageKeys * 128;                 // 8 KB per half-row tile
  static constexpr int kTensorStageBytes = kHalves * kHalfBytes;      // K (or V) per stage
  // bf16: ~96 KB in flight per CTA, two CTAs per SM; e4m3: 64 KB, three CTAs per SM (more
  // warps to hide the in-register conversions), six stages when the combine needs room
  static constexpr int kStages = KV8 ? (NT == 4 ? 6 : 4) : D == 128 ? 3 : 4;
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kStages * kTensorStageBytes;
  static constexpr int kPagesOff = 2 * kStages * kTensorStageBytes;
  static constexpr int kBarOff = (kPagesOff + kMaxItemPages * 4 + 127) / 128 * 128;
  static constexpr int kBytes = kBarOff + 2 * kStages * 8 + 16;
  static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1024
  // TMA destinations with 128-byte swizzle start on 1024-byte boundaries; mbarriers need 8.
  static_assert(kKOff % 1024 == 0 && kVOff % 1024 == 0 && kTensorStageBytes % 1024 == 0,
                "stage alignment");
  static_assert(kHalfBytes % 1024 == 0, "half-tile alignment");
  static_assert(kBarOff % 8 == 0, "mbarrier alignment");
  static_assert(!KV8 || D == 128, "e4m3 pools: head_dim 128");
  // the four warps' states are combined in the stage ring once it is drained
  static_assert(2 * kConsumerWarps * 8 * NT * 4 + kConsumerWarps * 8 * NT * (D + 4) * 4 <=
                    kPagesOff,
                "combine area");
};

struct alignas(16) U4 {
  uint32_t x, y, z, w;
};

template <int D, int NT, bool KV8>
__global__ void __launch_bounds__(kDecodeThreads, 1)
    decode_split_kernel(const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap vmap, DecodeLaunch p,
                        const __grid_constant__ DecodeItemsInline inl) {
  using Geo = DecodeGeom<D, KV8, NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* Ks = smem + Geo::kKOff;
  uint8_t* Vs = smem + Geo::kVOff;
  int32_t* pages = reinterpret_cast<int32_t*>(smem + Geo::kPagesOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Geo::kBarOff);
  uint64_t* empty = full + Geo::kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + Geo::kStages);
  volatile int* never = abort_flag + 1;  // stays 0: time-bounded waits that ignore an abort

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  // The grid is (KV heads, items), so that the CTAs of one item's KV heads start together and
  // read whole rows of sequence-major pages at once, or (items, KV heads) when the items pass
  // grid y's limit.  A square grid is read as the former: both readings visit every
  // (item, head) pair once.
  const bool heads_fast = (int)gridDim.x == p.num_kv_heads;
  const int item_idx = heads_fast ? (int)blockIdx.y : (int)blockIdx.x;
  if (p.count && item_idx >= __ldg(p.count)) return;  // device-planned: unused CTA
  const DecodeItem it = p.items ? p.items[item_idx] : inl.v[item_idx];
  const int h = heads_fast ? (int)blockIdx.x : (int)blockIdx.y;
  const int Hq = p.num_q_heads;
  const int G = Hq / p.num_kv_heads;
  const int rows = it.q_len * G;
  const int past = it.kv_len - it.q_len;
  const int nstages = (it.k_end - it.k_begin + Geo::kStageKeys - 1) / Geo::kStageKeys;
  const int P = p.kv.page_size;
  const int log2P = p.kv.log2_page;

  if (threadIdx.x == 0) {
    // the merge kernel (launched with programmatic dependent launch) may get its CTAs onto
    // the SMs now; it waits for this whole grid to finish before reading any partial result
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    for (int s = 0; s < Geo::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    *abort_flag = 0;
    *never = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---------------------------------------------------------------- producer warp
    const int first_blk = it.k_begin >> log2P;
    const int last_blk = (it.k_end - 1) >> log2P;
    const int npg = last_blk - first_blk + 1;
    const int32_t* bt_row =
        p.kv.layout == 0
            ? p.kv.block_table + (size_t)it.seq * p.kv.max_blocks
            : p.kv.block_table + ((size_t)it.seq * p.kv.num_kv_heads + h) * p.kv.max_blocks;
    for (int j = lane; j < npg; j += 32) pages[j] = __ldg(bt_row + first_blk + j);
    __syncwarp();
    if (p.k_new) {
      // fused KV write: the new tokens (positions past .. kv_len-1) that fall in this CTA's key
      // range are copied into their slots for KV head h before any page of the range is
      // loaded; the proxy fence orders these plain stores before the TMA reads below.
      const int lo = max(past, it.k_begin);
      const int ntok = it.k_end - lo;
      const int chunks = KV8 ? D / 16 : D / 8;  // 16-byte chunks per pool row
      for (int idx = lane; idx < 2 * ntok * chunks; idx += 32) {
        const int which = idx / (ntok * chunks);
        const int rem = idx - which * ntok * chunks;
        const int i = rem / chunks;
        const int c = rem - i * chunks;
        const int pos = lo + i;
        const int tok = it.t0 + (pos - past);
        const int page = pages[(pos >> log2P) - first_blk];
        if (page < 0 || page >= p.kv.num_pages) {
          atomicOr(p.err, kErrBadIndex);
          continue;
        }
        const size_t row = p.kv.layout == 0
                               ? ((size_t)page * P + (pos & (P - 1))) * p.num_kv_heads + h
                               : (size_t)page * P + (pos & (P - 1));
        if constexpr (KV8) {
          // 16 elements -> 16 codes: e4m3(fp32(x) / scale), nearest even, saturating
          const uint16_t* src = (which == 0 ? p.k_new : p.v_new) +
                                ((size_t)tok * p.num_kv_heads + h) * D + c * 16;
          const float sc = __ldg((which == 0 ? p.k_scale : p.v_scale) + h);
          uint8_t* dst = static_cast<uint8_t*>(which == 0 ? p.k_pool_w : p.v_pool_w) + row * D +
                         c * 16;
          *reinterpret_cast<uint4*>(dst) =
              e4m3_quantize16(__ldg(reinterpret_cast<const uint4*>(src)),
                              __ldg(reinterpret_cast<const uint4*>(src) + 1), sc);
        } else {
          const uint16_t* src = (which == 0 ? p.k_new : p.v_new) +
                                ((size_t)tok * p.num_kv_heads + h) * D + c * 8;
          uint16_t* dst = static_cast<uint16_t*>(which == 0 ? p.k_pool_w : p.v_pool_w) +
                          row * D + c * 8;
          *reinterpret_cast<uint4*>(dst) = __ldg(reinterpret_cast<const uint4*>(src));
        }
      }
      asm volatile("fence.proxy.async.global;" ::: "memory");
      __syncwarp();
    }
    if (lane == 0 && p.test_wait_ns == 0) {
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      const int hcoord = p.kv.layout == 0 ? h : 0;
      const int box_rows = P < Geo::kStageKeys ? P : Geo::kStageKeys;
      const uint32_t box_bytes = (uint32_t)box_rows * 128u;
      int issued = 0;
      for (int s = 0; s < nstages; ++s) {
        const int slot = s % Geo::kStages;
        if (s >= Geo::kStages &&
            !wait_bounded(&empty[slot], ((s / Geo::kStages) - 1) & 1, abort_flag, p.err,
                          kErrDecodeWait))
          break;
        const int kst = it.k_begin + s * Geo::kStageKeys;
        const int kend = min(kst + Geo::kStageKeys, it.k_end);
        const int b0 = kst >> log2P;
        const int b1 = (kend - 1) >> log2P;
        const int nbox = b1 - b0 + 1;
        mbar_arrive_expect_tx(&full[slot], 2u * Geo::kHalves * box_bytes * (uint32_t)nbox);
        for (int bi = 0; bi < nbox; ++bi) {
          const int blk = b0 + bi;
          const int page = pages[blk - first_blk];
          const int srow = P >= Geo::kStageKeys ? (kst & (P - 1)) : 0;
          const int drow = P >= Geo::kStageKeys ? 0 : blk * P - kst;
#pragma unroll
          for (int half = 0; half < Geo::kHalves; ++half) {
            const int off = slot * Geo::kTensorStageBytes + half * Geo::kHalfBytes + drow * 128;
            tma_load_4d(Ks + off, &kmap, half * 64, hcoord, srow, page, &full[slot]);
            tma_load_4d(Vs + off, &vmap, half * 64, hcoord, srow, page, &full[slot]);
          }
        }
        ++issued;
      }
      if (*abort_flag) {
        // let copies already in flight land before the CTA's shared memory goes away
        for (int s = max(0, issued - Geo::kStages); s < issued; ++s)
          wait_bounded(&full[s % Geo::kStages], (s / Geo::kStages) & 1, never, nullptr, 0,
                       kWaitTimeoutNs / 8);
      }
    }
    __syncwarp();
    return;  // the consumers keep the CTA (and its shared memory) alive until they finish
  } else {
    // ---------------------------------------------------------------- consumer warps
    constexpr int KT = D / 16;
    uint32_t bq[NT][KT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int col = nt * 8 + (lane >> 2);
      const bool ok = col < rows;
      const int tok = it.t0 + (ok ? col / G : 0);
      const int hq = h * G + (ok ? col % G : 0);
      const uint32_t* qrow =
          reinterpret_cast<const uint32_t*>(p.q + ((size_t)tok * Hq + hq) * D);
#pragma unroll
      for (int kk = 0; kk < KT; ++kk) {
        if constexpr (KV8) {
          // f16 operands; the head dims of a k-step are taken in the order that makes each
          // lane's K bytes contiguous: fragment columns (2t, 2t+1 | 2t+8, 2t+9) are dims
          // 16kk + 4t .. 4t+3 (the same order for Q and K leaves Q.K unchanged)
          bq[nt][kk][0] = ok ? bf16x2_to_f16x2(__ldg(qrow + kk * 8 + 2 * (lane & 3))) : 0u;
          bq[nt][kk][1] = ok ? bf16x2_to_f16x2(__ldg(qrow + kk * 8 + 2 * (lane & 3) + 1)) : 0u;
        } else {
          bq[nt][kk][0] = ok ? __ldg(qrow + kk * 8 + (lane & 3)) : 0u;
          bq[nt][kk][1] = ok ? __ldg(qrow + kk * 8 + 4 + (lane & 3)) : 0u;
        }
      }
    }
    float m[NT][2], ls[NT][2];
    float acc[KT][NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      m[nt][0] = m[nt][1] = -CUDART_INF_F;
      ls[nt][0] = ls[nt][1] = 0.f;
#pragma unroll
      for (int mt = 0; mt < KT; ++mt) acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] =
          acc[mt][nt][3] = 0.f;
    }
    // column -> visible-key limit (exclusive) for the causal mask
    int lim[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int col = nt * 8 + 2 * (lane & 3) + j;
        const int tok_i = col < rows ? col / G : 0;
        lim[nt][j] = p.causal ? min(it.k_end, past + tok_i + 1) : it.k_end;
      }

    // log2-domain score scale; e4m3 keys carry their KV head's scale (element = code * s)
    const float sl2 = KV8 ? p.scale_log2 * __ldg(p.k_scale + h) : p.scale_log2;
    const int ar = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;  // K ldmatrix row
    const int vr = warp * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;  // V ldmatrix.trans row
    for (int s = 0; s < nstages; ++s) {
      const int slot = s % Geo::kStages;
      if (!warp_wait_bounded(&full[slot], (s / Geo::kStages) & 1, abort_flag, p.err,
                             kErrDecodeWait, p.test_wait_ns ? p.test_wait_ns : kWaitTimeoutNs))
        break;
      const int key0 = it.k_begin + s * Geo::kStageKeys + warp * 16;
      if (key0 < it.k_end) {
        const uint32_t kbase = smem_u32(Ks + slot * Geo::kTensorStageBytes);
        float c[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) c[nt][0] = c[nt][1] = c[nt][2] = c[nt][3] = 0.f;
        if constexpr (KV8) {
          // key rows g and g + 8 of the warp's 16 (same swizzle phase); per k-step each lane
          // reads the 4 codes of dims 16kk + 4t .. 4t+3 of both rows
          const int rg = warp * 16 + (lane >> 2);
#pragma unroll
          for (int kk = 0; kk < KT; ++kk) {
            const uint32_t off = (uint32_t)(((kk ^ (rg & 7)) << 4) + 4 * (lane & 3));
            const uint32_t kg = ld_shared_u32(kbase + rg * 128 + off);
            const uint32_t kh = ld_shared_u32(kbase + (rg + 8) * 128 + off);
            const uint32_t a0 = e4m3x2_to_f16x2(kg), a2 = e4m3x2_to_f16x2(kg >> 16);
            const uint32_t a1 = e4m3x2_to_f16x2(kh), a3 = e4m3x2_to_f16x2(kh >> 16);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              mma_f16_16816(c[nt], a0, a1, a2, a3, bq[nt][kk][0], bq[nt][kk][1]);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < KT; ++kk) {
            const int chunk = 2 * kk + (lane >> 4);
            const uint32_t addr = kbase + (chunk >> 3) * Geo::kHalfBytes + ar * 128 +
                                  (((chunk & 7) ^ (ar & 7)) << 4);
            uint32_t a0, a1, a2, a3;
            ldsm_x4(addr, a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              mma_bf16_16816(c[nt], a0, a1, a2, a3, bq[nt][kk][0], bq[nt][kk][1]);
          }
        }
        const int k_lo = key0 + (lane >> 2);
        const int k_hi = k_lo + 8;
        uint32_t bp[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float pl[2], ph[2];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const float s_lo = k_lo < lim[nt][j] ? c[nt][j] * sl2 : -CUDART_INF_F;
            const float s_hi = k_hi < lim[nt][j] ? c[nt][2 + j] * sl2 : -CUDART_INF_F;
            float tmax = fmaxf(s_lo, s_hi);
            tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 4));
            tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 8));
            tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
            const float m_new = fmaxf(m[nt][j], tmax);
            const float m_use = m_new == -CUDART_INF_F ? 0.f : m_new;
            const float alpha = fast_exp2(m[nt][j] - m_use);
            pl[j] = fast_exp2(s_lo - m_use);
            ph[j] = fast_exp2(s_hi - m_use);
            ls[nt][j] = ls[nt][j] * alpha + pl[j] + ph[j];
            m[nt][j] = m_new;
#pragma unroll
            for (int mt = 0; mt < KT; ++mt) {
              acc[mt][nt][j] *= alpha;
              acc[mt][nt][2 + j] *= alpha;
            }
          }
          if constexpr (KV8) {
            bp[nt][0] = movmatrix_trans(pack_f16(pl[0], pl[1]));
            bp[nt][1] = movmatrix_trans(pack_f16(ph[0], ph[1]));
          } else {
            bp[nt][0] = movmatrix_trans(pack_bf16(pl[0], pl[1]));
            bp[nt][1] = movmatrix_trans(pack_bf16(ph[0], ph[1]));
          }
        }
        uint8_t* vtile = Vs + slot * Geo::kTensorStageBytes;
        const int nvalid = it.k_end - key0;
        if (nvalid < 16) {
          // rows past the last key may hold anything (NaN poison): P is 0 there, V must be 0
          const int nz = (16 - nvalid) * Geo::kHalves * 8;
          for (int i = lane; i < nz; i += 32) {
            const int row = nvalid + i / (Geo::kHalves * 8);
            const int rem = i % (Geo::kHalves * 8);
            *reinterpret_cast<U4*>(vtile + (rem >> 3) * Geo::kHalfBytes +
                                   (warp * 16 + row) * 128 + (rem & 7) * 16) = U4{0, 0, 0, 0};
          }
          __syncwarp();
        }
        const uint32_t vbase = smem_u32(vtile);
        if constexpr (KV8) {
          // V^T as the A operand from e4m3 rows: a transposing 8x8 load of byte pairs gives
          // lane (g, t) the codes of dims 2g, 2g+1 of keys 2t, 2t+1; byte permutes split them
          // into the (keys 2t, 2t+1) pairs of dim 2g (fragment row g) and of dim 2g+1 (row
          // g + 8), so M-tile mt holds dims 16mt + 2r (rows r < 8) and 16mt + 2(r-8) + 1
          const int vrow = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
          for (int mt = 0; mt < KT; mt += 2) {
            const int chunk = mt + (lane >> 4);
            const uint32_t addr = vbase + vrow * 128 + (((chunk & 7) ^ (vrow & 7)) << 4);
            uint32_t r0, r1, r2, r3;
            ldsm_x4_trans(addr, r0, r1, r2, r3);
            const uint32_t x0 = e4m3x2_to_f16x2(__byte_perm(r0, 0, 0x0020));
            const uint32_t x1 = e4m3x2_to_f16x2(__byte_perm(r0, 0, 0x0031));
            const uint32_t x2 = e4m3x2_to_f16x2(__byte_perm(r1, 0, 0x0020));
            const uint32_t x3 = e4m3x2_to_f16x2(__byte_perm(r1, 0, 0x0031));
            const uint32_t y0 = e4m3x2_to_f16x2(__byte_perm(r2, 0, 0x0020));
            const uint32_t y1 = e4m3x2_to_f16x2(__byte_perm(r2, 0, 0x0031));
            const uint32_t y2 = e4m3x2_to_f16x2(__byte_perm(r3, 0, 0x0020));
            const uint32_t y3 = e4m3x2_to_f16x2(__byte_perm(r3, 0, 0x0031));
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              mma_f16_16816(acc[mt][nt], x0, x1, x2, x3, bp[nt][0], bp[nt][1]);
              mma_f16_16816(acc[mt + 1][nt], y0, y1, y2, y3, bp[nt][0], bp[nt][1]);
            }
          }
        } else {
#pragma unroll
          for (int mt = 0; mt < KT; ++mt) {
            const int chunk = 2 * mt + ((lane >> 3) & 1);
            const uint32_t addr = vbase + (chunk >> 3) * Geo::kHalfBytes + vr * 128 +
                                  (((chunk & 7) ^ (vr & 7)) << 4);
            uint32_t a0, a1, a2, a3;
            ldsm_x4_trans(addr, a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              mma_bf16_16816(acc[mt][nt], a0, a1, a2, a3, bp[nt][0], bp[nt][1]);
          }
        }
        if (nvalid < 16) fence_proxy_async_smem();  // generic writes before the next TMA
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }
    // row sums: reduce the per-lane partials over the 8 lanes of each column
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float v = ls[nt][j];
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        ls[nt][j] = v;
      }
    // every consumer warp has waited on every stage, so all copies have landed; once all
    // four are done reading, the stage ring is free for the combine
    asm volatile("bar.sync 1, 128;" ::: "memory");
    // --------------------------------------------- combine the four warps (reuse K ring)
    constexpr int COLS = 8 * NT;
    constexpr int OPAD = D + 4;
    float* red_m = reinterpret_cast<float*>(smem);
    float* red_l = red_m + kConsumerWarps * COLS;
    float* red_o = red_l + kConsumerWarps * COLS;
    if (!*abort_flag) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int col = nt * 8 + 2 * (lane & 3) + j;
          if ((lane >> 2) == 0) {
            red_m[warp * COLS + col] = m[nt][j];
            red_l[warp * COLS + col] = ls[nt][j];
          }
          float* o = red_o + (warp * COLS + col) * OPAD;
#pragma unroll
          for (int mt = 0; mt < KT; ++mt) {
            if constexpr (KV8) {  // fragment rows r, r + 8 are dims 16mt + 2r, 16mt + 2r + 1
              o[mt * 16 + 2 * (lane >> 2)] = acc[mt][nt][j];
              o[mt * 16 + 2 * (lane >> 2) + 1] = acc[mt][nt][2 + j];
            } else {
              o[mt * 16 + (lane >> 2)] = acc[mt][nt][j];
              o[mt * 16 + (lane >> 2) + 8] = acc[mt][nt][2 + j];
            }
          }
        }
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (!*abort_flag) {
      const int Hkv = p.num_kv_heads;
      const float vsc = KV8 ? __ldg(p.v_scale + h) : 1.f;  // e4m3 V: element = code * scale
      for (int idx = threadIdx.x; idx < rows * D; idx += kConsumerWarps * 32) {
        const int col = idx / D;
        const int d = idx - col * D;
        float M = -CUDART_INF_F;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, red_m[w * COLS + col]);
        float L = 0.f, O = 0.f;
        if (M != -CUDART_INF_F) {
#pragma unroll
          for (int w = 0; w < kConsumerWarps; ++w) {
            const float f = fast_exp2(red_m[w * COLS + col] - M);
            L += red_l[w * COLS + col] * f;
            O += red_o[(w * COLS + col) * OPAD + d] * f;
          }
        }
        const float o = L > 0.f ? O / L * vsc : 0.f;
        const float lse2 = L > 0.f ? M + fast_log2(L) : -CUDART_INF_F;
        const int tok = it.t0 + col / G;
        const int hq = h * G + col % G;
        if (it.part_slot < 0) {
          const __nv_bfloat16 ob = __float2bfloat16_rn(o);
          p.out[((size_t)tok * Hq + hq) * D + d] = *reinterpret_cast<const uint16_t*>(&ob);
          if (d == 0 && p.lse) p.lse[(size_t)tok * Hq + hq] = lse2 * 0.69314718055994531f;
        } else {
          const size_t prow = ((size_t)it.part_slot * Hkv + h) * p.rows_per_item + col;
          p.part_o[prow * D + d] = o;
          if (d == 0) p.part_lse[prow] = lse2;
        }
      }
    }
  }
}

template <int D>
__global__ void __launch_bounds__(128) merge_kernel(MergeLaunch p,
                                                    const __grid_constant__ MergeRowsInline inl) {
  // launched early (programmatic dependent launch): wait until the decode grid has finished
  // and its partial results are visible
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int gw = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int Hq = p.num_q_heads;
  const int nrows = p.count ? __ldg(p.count) : p.num_rows;
  if (gw >= nrows * Hq) return;
  const int r = gw / Hq;
  const int hq = gw - r * Hq;
  const int G = Hq / p.num_kv_heads;
  const MergeRow mr = p.rows ? p.rows[r] : inl.v[r];
  const int h = hq / G;
  const int col = mr.local * G + (hq - h * G);
  constexpr int E = D / 32;
  float M = -CUDART_INF_F;
  for (int s = 0; s < mr.nsplit; ++s) {
    const size_t prow = ((size_t)(mr.first_slot + s) * p.num_kv_heads + h) * p.rows_per_item + col;
    M = fmaxf(M, p.part_lse[prow]);
  }
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  float W = 0.f;
  if (M != -CUDART_INF_F) {
    for (int s = 0; s < mr.nsplit; ++s) {
      const size_t prow =
          ((size_t)(mr.first_slot + s) * p.num_kv_heads + h) * p.rows_per_item + col;
      const float l = p.part_lse[prow];
      const float w = l == -CUDART_INF_F ? 0.f : fast_exp2(l - M);
      W += w;
      const float* po = p.part_o + prow * D;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] += w * po[e * 32 + lane];
    }
  }
  const float inv = W > 0.f ? 1.f / W : 0.f;
  uint16_t* o = p.out + ((size_t)mr.token * Hq + hq) * D;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const __nv_bfloat16 ob = __float2bfloat16_rn(acc[e] * inv);
    o[e * 32 + lane] = *reinterpret_cast<const uint16_t*>(&ob);
  }
  if (lane == 0 && p.lse)
    p.lse[(size_t)mr.token * Hq + hq] =
        W > 0.f ? (M + fast_log2(W)) * 0.69314718055994531f : -CUDART_INF_F;
}

template <int D, int NT, bool KV8>
cudaError_t launch_decode_t(const DecodeLaunch& p, const DecodeItemsInline* inl,
                            cudaStream_t stream) {
  using Geo = DecodeGeom<D, KV8, NT>;
  // 4-D box over the pool: (dims, kv head, slot, page); head-major pools use one "head".
  CUtensorMap kmap, vmap;
  cudaError_t e = encode_kv_map(&kmap, p.kv.k_pool, p.kv, D, kDecodeStageKeys);
  if (e != cudaSuccess) return e;
  e = encode_kv_map(&vmap, p.kv.v_pool, p.kv, D, kDecodeStageKeys);
  if (e != cudaSuccess) return e;
  auto kern = decode_split_kernel<D, NT, KV8>;
  e = ensure_smem_attr(reinterpret_cast<const void*>(kern), Geo::kAlloc);
  if (e != cudaSuccess) return e;
  const dim3 grid = p.num_items <= 65535 ? dim3(p.num_kv_heads, p.num_items)
                                         : dim3(p.num_items, p.num_kv_heads);
  kern<<<grid, kDecodeThreads, Geo::kAlloc, stream>>>(kmap, vmap, p, *inl);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeLaunch& p, const DecodeItemsInline* inl, int nt,
                          cudaStream_t stream) {
  if (p.num_items <= 0) return cudaSuccess;
  if (p.kv.kv8) {
    if (p.head_dim != 128) return cudaErrorInvalidValue;
    if (nt == 1) return launch_decode_t<128, 1, true>(p, inl, stream);
    if (nt == 2) return launch_decode_t<128, 2, true>(p, inl, stream);
    return launch_decode_t<128, 4, true>(p, inl, stream);
  }
  if (p.head_dim == 128) {
    if (nt == 1) return launch_decode_t<128, 1, false>(p, inl, stream);
    if (nt == 2) return launch_decode_t<128, 2, false>(p, inl, stream);
    return launch_decode_t<128, 4, false>(p, inl, stream);
  }
  if (nt == 1) return launch_decode_t<64, 1, false>(p, inl, stream);
  if (nt == 2) return launch_decode_t<64, 2, false>(p, inl, stream);
  return launch_decode_t<64, 4, false>(p, inl, stream);
}

cudaError_t launch_merge(const MergeLaunch& p, const MergeRowsInline* inl, cudaStream_t stream) {
  if (p.num_rows <= 0) return cudaSuccess;
  const long warps = (long)p.num_rows * p.num_q_heads;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((warps + 3) / 4));
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (p.head_dim == 128) return cudaLaunchKernelEx(&cfg, merge_kernel<128>, p, *inl);
  return cudaLaunchKernelEx(&cfg, merge_kernel<64>, p, *inl);
}

}  // namespace rpa
