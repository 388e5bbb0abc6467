// Causal paged prefill on the 5th-generation tensor cores (tcgen05 + TMEM), fed by TMA through
// the block table; also the sparse mode that walks per-group block tables.
//
// What it computes: for a tile of 128 query tokens of one sequence and one query head, exact
// softmax attention over the keys the tokens may see -- 0 .. past + i when causal (bottom-right
// alignment: "[WebGPU] Optimized PagedAttention implementation (2/n)", commit "FlashAttention:
// optional seqlens_q input"), restricted in sparse mode to the KV blocks listed in the table of
// the head's KV group ("CompactAttention: Accelerating Chunked Prefill with Block-Union KV
// Selection", Fig. 3: the paged kernel reads the selected pages in place).  This is the fused
// paged prefill of the WebGPU page ("What's shipped": FlashAttentionPagedPrefillProgram, one
// block-table lookup per K/V tile) and the prefill specialisation of "Ragged Paged Attention:
// A High-Performance and Flexible LLM Inference Kernel for TPU" (Key ideas).
//
// B200 design.  The work comes in units of (128-query tile, pair of query heads of one KV
// group) -- the two heads share every K/V tile and the same causal mask.  A persistent CTA
// holds one SM (all 512 TMEM columns) and walks its share of the units, so the next unit's Q,
// K and V stream in, and its first S is computed, while the current unit's O is written out.
// Beside a decode kernel (mixed batches, device-planned steps) the grid has one CTA per unit
// instead, so that decode CTAs take SMs as units finish.
// 384 threads:
//   warp 0      TMA producer: both Q tiles of a unit, then K and V tiles of 128 keys, page by
//               page (boxes of [min(P,128) slots x 64 dims], 128-byte swizzle), 2-stage ring;
//   warp 1      allocates TMEM; one thread issues the MMAs, interleaving the two heads so the
//               tensor pipe works on one head while the other head's softmax runs:
//                 S_h = Q_h K_j^T   (M=128 queries, N=128 keys, K=D; SMEM descriptors)
//                 O_h += P_h V_j    (M=128, N=D, K=128 keys; P_h read from TMEM, V MN-major)
//   warps 4-7   softmax of head A, warps 8-11 softmax of head B: thread r owns query row r
//               (TMEM lane r); it loads S, masks, takes exp2 against a reference max, writes P
//               as bf16 over S and arrives.  The reference max is set by the first tile that
//               shows the row a key and then held (no max pass per tile); only a tile whose row
//               sum would pass 2^64 moves it, and only then is O rescaled in TMEM (after the
//               previous P.V finished), so the softmax never waits on P.V otherwise.
// TMEM columns: S_A [0,128) S_B [128,256) O_A [256,256+D) O_B [384,384+D).  Bounded waits.
// An odd GQA group size runs with head B switched off.
// e4m3 pools (kKv8): the K/V boxes bring one-byte codes into the upper half of their slot;
// warps 2-3 expand each row in place to f16 (e4m3 -> f16 is exact) and convert the unit's Q
// from bf16 to f16 (exact in f16's range), so the MMAs run kind::f16 on f16 operands.  P is
// then written as f16, whose range ends at 65504, so a tile is redone once its row sum passes
// 2^15 instead of 2^64.  The score scale carries the KV head's k_scale, the output its v_scale.
#include <cuda_bf16.h>
#include <type_traits>
#include <math_constants.h>

#include "ptx.cuh"
#include "rpa_internal.h"

namespace rpa {
namespace {

constexpr int kThreads = 384;
constexpr int kStagesK = 2;  // K tiles in flight
constexpr int kStagesV = 2;  // V tiles in flight
constexpr int kRows = kPrefillTileRows;  // 128
static_assert(kRows == 128, "query-tile table rows are q_start >> 7");
constexpr int kKeys = kPrefillTileKeys;  // 128
constexpr uint32_t kTmemCols = 512;
constexpr float kMaxTileSum = 0x1p64f;    // a tile whose row sum passes this is redone
constexpr float kMaxTileSumF16 = 0x1p15f;  // the same with P as f16 (e4m3 pools)
// Registers: the CTA launches with kLaunchRegs per thread (3 warpgroups); the producer/MMA
// warpgroup gives most of its share to the two softmax warpgroups.
constexpr int kLaunchRegs = 168;
constexpr int kRegsControl = 64;
constexpr int kRegsSoftmax = 216;
static_assert(kRegsControl + 2 * kRegsSoftmax <= 3 * kLaunchRegs, "register split");

template <int D>
struct PfGeom {
  static constexpr int kHalves = D / 64;
  static constexpr int kHalfBytes = 128 * 128;             // 128 rows x 128 B
  static constexpr int kTileBytes = kHalves * kHalfBytes;  // a Q, K or V tile
  static constexpr int kQOff = 0;                          // Q_A, Q_B
  static constexpr int kKOff = 2 * kTileBytes;
  static constexpr int kVOff = kKOff + kStagesK * kTileBytes;
  static constexpr int kBarOff = kVOff + kStagesV * kTileBytes;
  // q_full, k_full[S], v_full[S], k_empty[S], v_empty[S], s_full[2], p_ready[2], o_done[2],
  // q_empty, mma_done, q_conv, k_conv[S], v_conv[S]
  static constexpr int kNumBars = 1 + 2 * kStagesK + 2 * kStagesV + 6 + 2 + 1 + kStagesK + kStagesV;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 64;
  // at least 120 KB so that a second CTA never shares the SM (and its 512 TMEM columns)
  static constexpr int kAlloc = kBytes + 1024 > 120 * 1024 ? kBytes + 1024 : 120 * 1024;
  static_assert(kKOff % 1024 == 0 && kVOff % 1024 == 0 && kTileBytes % 1024 == 0,
                "TMA destinations with 128-byte swizzle start on 1024-byte boundaries");
  static_assert(kBarOff % 8 == 0 && kMiscOff % 8 == 0, "mbarrier alignment");
  static_assert(kAlloc <= 227 * 1024, "shared memory per CTA");
};

struct alignas(16) U4 {
  uint32_t x, y, z, w;
};

// Number of entries of the ascending list t[0, n) that are below `limit`, found by the whole
// warp: each round probes 32 evenly spaced entries at once and keeps the one gap where the
// answer lies, so a 2048-entry table takes three dependent loads instead of eleven.
__device__ __forceinline__ int warp_count_below(const int32_t* t, int n, int limit) {
  const int lane = threadIdx.x & 31;
  int lo = 0, hi = n;  // t[i] < limit for i < lo; t[i] >= limit for i >= hi
  while (hi - lo > 32) {
    const int step = (hi - lo + 32) / 33;
    const int idx = lo + (lane + 1) * step;
    const bool below = idx < hi && __ldg(t + idx) < limit;
    const int c = __popc(__ballot_sync(0xffffffffu, below));
    const int nlo = c > 0 ? lo + c * step + 1 : lo;
    const int nhi = (c < 32 && lo + (c + 1) * step < hi) ? lo + (c + 1) * step : hi;
    lo = nlo;
    hi = nhi;
  }
  const bool below = lo + lane < hi && __ldg(t + lo + lane) < limit;
  return lo + __popc(__ballot_sync(0xffffffffu, below));
}

// One unit of work: a 128-query tile of one sequence and the pair (or single head) of query
// heads it serves, with the key tiles those rows see.
struct Unit {
  PrefillTile tile;
  int hq0, h;            // first query head, KV head
  int past, kv_hi;       // context before the chunk; keys [0, kv_hi) are visible to the tile
  const int32_t* table;  // sparse modes: the table row, else null
  int n_entries;         // sparse modes: table entries before kv_hi
  int n_tiles;           // 128-key tiles
};

template <int D, bool kFuse, bool kKv8>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap qmap,
                   const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap,
                   const __grid_constant__ CUtensorMap knmap,
                   const __grid_constant__ CUtensorMap vnmap, PrefillLaunch p,
                   const __grid_constant__ PrefillTilesInline inl) {
  using Geo = PfGeom<D>;
  static_assert(!(kFuse && kKv8), "the fused KV write is for bf16 pools");
  static_assert(!kKv8 || D == 128, "e4m3 pools: head_dim 128");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* Qs = smem + Geo::kQOff;
  uint8_t* Ks = smem + Geo::kKOff;
  uint8_t* Vs = smem + Geo::kVOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Geo::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + kStagesK;
  uint64_t* k_empty = v_full + kStagesV;   // K slot free: both heads' S MMAs done
  uint64_t* v_empty = k_empty + kStagesK;  // V slot free: both heads' P.V MMAs done
  uint64_t* s_full = v_empty + kStagesV;   // [2] per head
  uint64_t* p_ready = s_full + 2;           // [2]
  uint64_t* o_done = p_ready + 2;           // [2]
  uint64_t* q_empty = o_done + 2;           // the unit's S MMAs are done with Q
  uint64_t* mma_done = q_empty + 1;
  // e4m3 pools: the f16 operands are ready (one arrival per converting warp)
  uint64_t* q_conv = mma_done + 1;
  uint64_t* k_conv = q_conv + 1;           // [kStagesK]
  uint64_t* v_conv = k_conv + kStagesK;    // [kStagesV]
  uint32_t* tmem_base_sh = reinterpret_cast<uint32_t*>(smem + Geo::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Geo::kMiscOff + 8);
  volatile int* never = reinterpret_cast<volatile int*>(smem + Geo::kMiscOff + 12);  // stays 0

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int Hq = p.num_q_heads;
  const int G = Hq / p.num_kv_heads;
  // query heads per unit: a pair of one KV group (they share every K/V tile); one head with
  // per-(query tile, head) tables or an odd group size
  const int hpc = (p.qtile_table == nullptr && (G & 1) == 0) ? 2 : 1;
  const int groups = Hq / hpc;
  const int n_list = p.count ? min(__ldg(p.count), p.num_tiles) : p.num_tiles;
  const int num_units = n_list * groups;
  const int P = p.kv.page_size;
  const int log2P = p.kv.log2_page;
  if ((int)blockIdx.x >= num_units) return;  // no unit at all (device-planned step)

  // The CTA walks units in rounds of gridDim.x, left to right in even rounds and right to left
  // in odd ones: the list is sorted heaviest first, so the alternation evens out the SMs' load.
  auto unit_index = [&](int k) {
    const int base = k * (int)gridDim.x;
    return (k & 1) ? base + (int)gridDim.x - 1 - (int)blockIdx.x : base + (int)blockIdx.x;
  };
  // every role walks the same units and counts barrier phases itself; called by whole warps
  // (the table search is warp-cooperative)
  auto unit_at = [&](int u) {
    Unit w;
    const int tile_idx = u / groups;
    w.hq0 = (u - tile_idx * groups) * hpc;
    w.tile = p.tiles ? p.tiles[tile_idx] : inl.v[tile_idx];
    w.h = w.hq0 / G;
    w.past = w.tile.kv_len - w.tile.q_len;
    const int q_end = min(w.tile.q_len, w.tile.q_start + kRows);  // local, exclusive
    w.kv_hi = p.causal ? min(w.tile.kv_len, w.past + q_end) : w.tile.kv_len;
    // key tiles: dense -> ceil(kv_hi/128); sparse -> visible table entries, 128/P per tile
    w.table = nullptr;
    w.n_entries = 0;
    if (p.group_table || p.qtile_table) {
      // the table of the pair's KV group, or of this query tile and head
      const size_t row = p.qtile_table ? ((size_t)w.tile.seq * Hq + w.hq0) * p.qtiles_per_seq +
                                             (w.tile.q_start >> 7)
                                       : (size_t)w.tile.seq * p.num_kv_heads + w.h;
      w.table = (p.qtile_table ? p.qtile_table : p.group_table) + row * p.kv.max_blocks;
      const int cnt =
          min(__ldg((p.qtile_table ? p.qtile_count : p.group_count) + row), p.kv.max_blocks);
      // entries (ascending block ids) whose block starts before kv_hi
      w.n_entries = warp_count_below(w.table, max(cnt, 0), (w.kv_hi + P - 1) >> log2P);
      const int per = kKeys >> log2P;
      w.n_tiles = (w.n_entries + per - 1) / per;
    } else {
      w.n_tiles = (w.kv_hi + kKeys - 1) / kKeys;
    }
    return w;
  };
  // rows of key tile j that hold real keys of the sequence (the rest of the slot is stale or
  // a tail past the sequence end)
  auto valid_keys = [&](const Unit& w, int j) {
    if (w.table) {
      const int per = kKeys >> log2P;
      const int ne = min(per, w.n_entries - j * per);
      const int last = __ldg(w.table + j * per + ne - 1);
      return (ne - 1) * P + min(P, w.tile.kv_len - (last << log2P));
    }
    const int covered = min(w.tile.kv_len, ((w.kv_hi + P - 1) >> log2P) << log2P);
    return min(kKeys, covered - j * kKeys);
  };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < kStagesK; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < kStagesV; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&p_ready[x], 128);
      mbar_init(&o_done[x], 1);
    }
    mbar_init(mma_done, 1);
    mbar_init(q_conv, 2);
    for (int s = 0; s < kStagesK; ++s) mbar_init(&k_conv[s], 2);
    for (int s = 0; s < kStagesV; ++s) mbar_init(&v_conv[s], 2);
    *abort_flag = 0;
    *never = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_sh;

  // Registers are rebalanced at the top of each warpgroup's branch: the control warpgroup
  // (producer, MMA issuer, two idle warps) gives registers to the softmax warpgroups, whose
  // threads each hold a 128-value S row.
  if (warp < 4) {
    regs_dealloc<kRegsControl>();
  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    // the whole warp walks the units; lane 0 issues the copies and keeps the counters
    if (lane == 0) {
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      if (kFuse && p.fuse_rows > 0) {
        tma_prefetch_desc(&knmap);
        tma_prefetch_desc(&vnmap);
      }
    }
    int kv_iter = 0;         // K/V tiles begun, over all units of this CTA
    int q_iter = 0;          // Q tiles begun
    int issued[2] = {0, 0};  // K and V tiles whose copies were started
    bool stop = false;
    for (int k = 0; !stop; ++k) {
      const int u = unit_index(k);
      if (u >= num_units) break;
      const Unit w = unit_at(u);
      if (w.n_tiles == 0) continue;
      if (lane == 0) {
        // Q of the previous unit stays until its S MMAs are done
        if (q_iter > 0 &&
            !wait_bounded(q_empty, (q_iter - 1) & 1, abort_flag, p.err, kErrPrefillWait))
          stop = true;
        if (!stop) {
          mbar_arrive_expect_tx(q_full, Geo::kTileBytes * hpc);
          for (int x = 0; x < hpc; ++x)
#pragma unroll
            for (int half = 0; half < Geo::kHalves; ++half)
              tma_load_3d(Qs + x * Geo::kTileBytes + half * Geo::kHalfBytes, &qmap, half * 64,
                          w.hq0 + x, w.tile.t0 + w.tile.q_start, q_full);
          ++q_iter;
        }
        const int32_t* bt_row =
            p.kv.layout == 0
                ? p.kv.block_table + (size_t)w.tile.seq * p.kv.max_blocks
                : p.kv.block_table +
                      ((size_t)w.tile.seq * p.kv.num_kv_heads + w.h) * p.kv.max_blocks;
        const int hcoord = p.kv.layout == 0 ? w.h : 0;
        const int box_rows = P < kKeys ? P : kKeys;
        // first key position served from k_new / v_new (-1: none)
        const int fuse_edge =
            kFuse && p.fuse_rows > 0 ? (w.past + p.fuse_rows - 1) / p.fuse_rows * p.fuse_rows
                                     : -1;
        // bf16: two 128-byte halves per row; e4m3: one 128-byte run of codes per row, into
        // the slot's upper half (expanded to f16 in place by the converting warps)
        constexpr int kLoads = kKv8 ? 1 : Geo::kHalves;
        constexpr int kDst0 = kKv8 ? Geo::kHalfBytes : 0;
        const uint32_t box_bytes = (uint32_t)box_rows * 128u * kLoads;
        for (int j = 0; !stop && j < w.n_tiles; ++j) {
          const int it = kv_iter++;
          int nbox, first_blk = 0, slot0 = 0;
          if (w.table) {
            nbox = min(kKeys >> log2P, w.n_entries - j * (kKeys >> log2P));
          } else if (P >= kKeys) {
            nbox = 1;
            first_blk = (j * kKeys) >> log2P;
            slot0 = (j * kKeys) & (P - 1);
          } else {
            first_blk = (j * kKeys) >> log2P;
            nbox = ((min(j * kKeys + kKeys, w.kv_hi) - 1) >> log2P) - first_blk + 1;
          }
          // A tile holding keys at or past fuse_edge (this step's new rows, read from k_new /
          // v_new; the pool gets them from the writer warps of this launch) takes the loop
          // below that decides per box; every other tile the plain pool loop.
          const bool tile_new =
              kFuse && fuse_edge >= 0 && (w.table ? true : j * kKeys + kKeys > fuse_edge);
          // K first (S needs it first), then V; each waits for its own slot to be released
          for (int kv = 0; kv < 2; ++kv) {
            const int ns = kv == 0 ? kStagesK : kStagesV;
            const int slot = it % ns;
            uint64_t* empty = kv == 0 ? &k_empty[slot] : &v_empty[slot];
            if (it >= ns && !wait_bounded(empty, ((it / ns) - 1) & 1, abort_flag, p.err,
                                          kErrPrefillWait)) {
              stop = true;
              break;
            }
            mbar_arrive_expect_tx(kv == 0 ? &k_full[slot] : &v_full[slot], box_bytes * nbox);
            uint8_t* dst_base = (kv == 0 ? Ks : Vs) + slot * Geo::kTileBytes;
            const CUtensorMap* map = kv == 0 ? &kmap : &vmap;
            uint64_t* bar = kv == 0 ? &k_full[slot] : &v_full[slot];
            if (tile_new) {
              for (int i = 0; i < nbox; ++i) {
                const int blk =
                    w.table ? __ldg(w.table + j * (kKeys >> log2P) + i) : first_blk + i;
                const int kst = (blk << log2P) + slot0;
                uint8_t* dst = dst_base + i * box_rows * 128;
                if (blk >= 0 && blk < p.kv.max_blocks && kst >= fuse_edge) {
                  const CUtensorMap* nmap = kv == 0 ? &knmap : &vnmap;
#pragma unroll
                  for (int half = 0; half < Geo::kHalves; ++half)
                    tma_load_3d(dst + half * Geo::kHalfBytes, nmap, half * 64, w.h,
                                w.tile.t0 + (kst - w.past), bar);
                } else {
                  int page = -1;
                  if (blk >= 0 && blk < p.kv.max_blocks)
                    page = __ldg(bt_row + blk);
                  else if (kv == 0)
                    atomicOr(p.err, kErrBadIndex);
#pragma unroll
                  for (int half = 0; half < Geo::kHalves; ++half)
                    tma_load_4d(dst + half * Geo::kHalfBytes, map, half * 64, hcoord, slot0,
                                page, bar);
                }
              }
            } else
            for (int i = 0; i < nbox; ++i) {
              const int blk =
                  w.table ? __ldg(w.table + j * (kKeys >> log2P) + i) : first_blk + i;
              int page = -1;  // out-of-range coordinates make TMA fill zeros: no stray access
              if (blk >= 0 && blk < p.kv.max_blocks)
                page = __ldg(bt_row + blk);
              else if (kv == 0)
                atomicOr(p.err, kErrBadIndex);
#pragma unroll
              for (int half = 0; half < kLoads; ++half)
                tma_load_4d(dst_base + kDst0 + half * Geo::kHalfBytes + i * box_rows * 128, map,
                            half * 64, hcoord, slot0, page, bar);
            }
            issued[kv] = it + 1;
          }
        }
      }
      stop = __shfl_sync(0xffffffffu, stop, 0);
    }
    if (lane == 0 && *abort_flag) {
      // let copies in flight land before shared memory goes away (time-bounded only: the
      // raised abort flag must not cut these waits short)
      if (q_iter > 0)
        wait_bounded(q_full, (q_iter - 1) & 1, never, nullptr, 0, kWaitTimeoutNs / 8);
      for (int kv = 0; kv < 2; ++kv) {
        const int ns = kv == 0 ? kStagesK : kStagesV;
        for (int i = max(0, issued[kv] - ns); i < issued[kv]; ++i)
          wait_bounded(kv == 0 ? &k_full[i % ns] : &v_full[i % ns], (i / ns) & 1, never,
                       nullptr, 0, kWaitTimeoutNs / 8);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_s = kKv8 ? idesc_f16_f32(128, kKeys, false, false)
                                      : idesc_bf16_f32(128, kKeys, false, false);
    constexpr uint32_t idesc_o =
        kKv8 ? idesc_f16_f32(128, D, false, true) : idesc_bf16_f32(128, D, false, true);
    // operands are ready: TMA done (bf16), or converted to f16 (e4m3 pools)
    uint64_t* const q_in = kKv8 ? q_conv : q_full;
    uint64_t* const k_in = kKv8 ? k_conv : k_full;
    uint64_t* const v_in = kKv8 ? v_conv : v_full;
    // Descriptors are built once; an MMA's operands differ from the base only in the start
    // address field (bits 0..13, in 16-byte units, no carry for addresses below 256 KB), so
    // each MMA needs one add per operand instead of rebuilding a 64-bit descriptor.
    const uint64_t dq0 = smem_desc_sw128(smem_u32(Qs), 16, 1024);
    const uint64_t dk0 = smem_desc_sw128(smem_u32(Ks), 16, 1024);
    const uint64_t dv0 = smem_desc_sw128(smem_u32(Vs), Geo::kHalfBytes, 1024);
    auto issue_s = [&](int x, int it) {  // S_x = Q_x K^T (K tile `it`) into TMEM [128x, +128)
      const uint32_t a_lo = (uint32_t)dq0 + (uint32_t)((x * Geo::kTileBytes) >> 4);
      const uint32_t b_lo =
          (uint32_t)dk0 + (uint32_t)(((it % kStagesK) * Geo::kTileBytes) >> 4);
      const uint32_t a_hi = (uint32_t)(dq0 >> 32), b_hi = (uint32_t)(dk0 >> 32);
      const uint32_t d = tmem + x * 128;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (uint32_t)(((kk >> 2) * Geo::kHalfBytes + (kk & 3) * 32) >> 4);
        if (kk == 0) umma_ss_lh<0>(d, a_lo + off, a_hi, b_lo + off, b_hi, idesc_s);
        else umma_ss_lh<1>(d, a_lo + off, a_hi, b_lo + off, b_hi, idesc_s);
      }
      umma_commit(&s_full[x]);
    };
    auto issue_o = [&](int x, int it, bool first) {  // O_x (+)= P_x V (V tile `it`)
      const uint32_t b_lo =
          (uint32_t)dv0 + (uint32_t)(((it % kStagesV) * Geo::kTileBytes) >> 4);
      const uint32_t b_hi = (uint32_t)(dv0 >> 32);
      const uint32_t d = tmem + 256 + x * 128;
      const uint32_t a = tmem + x * 128;
      const uint32_t acc0 = first ? 0u : 1u;
#pragma unroll
      for (int kk = 0; kk < kKeys / 16; ++kk)
        umma_ts_lh(d, a + kk * 8, b_lo + (uint32_t)((kk * 2048) >> 4), b_hi, idesc_o,
                   kk > 0 ? 1u : acc0);
      umma_commit(&o_done[x]);
    };
    bool ok = true;
    int kv_iter = 0;  // K/V tiles consumed, over all units of this CTA
    int q_iter = 0;   // units with key tiles
    for (int k = 0; ok; ++k) {
      const int u = unit_index(k);
      if (u >= num_units) break;
      const Unit w = unit_at(u);
      if (w.n_tiles == 0) continue;
      // The unit's first S goes in as soon as its Q and first K tile are in: the softmax
      // warps are still writing out the previous unit's O (the first P.V of this unit, which
      // overwrites O, waits for their P, which they produce only after that).
      ok = warp_wait_bounded(q_in, q_iter & 1, abort_flag, p.err, kErrPrefillWait) &&
           warp_wait_bounded(&k_in[kv_iter % kStagesK], (kv_iter / kStagesK) & 1,
                             abort_flag, p.err, kErrPrefillWait);
      ++q_iter;
      if (!ok) break;
      if (lane == 0) {
        tc_fence_after();
        for (int x = 0; x < hpc; ++x) issue_s(x, kv_iter);
        umma_commit(&k_empty[kv_iter % kStagesK]);  // free once both S MMAs finish
        if (w.n_tiles == 1) umma_commit(q_empty);    // the unit's last S
      }
      __syncwarp();
      for (int j = 0; ok && j < w.n_tiles; ++j) {
        const int it = kv_iter + j;
        const int slot = it % kStagesV;
        if (!warp_wait_bounded(&v_in[slot], (it / kStagesV) & 1, abort_flag, p.err,
                               kErrPrefillWait)) {
          ok = false;
          break;
        }
        // V rows past the last real key may hold anything (NaN tail slots, a stale tile):
        // P = 0 there does not cancel a NaN in the product, so the rows are zeroed (by the
        // converting warps for e4m3 pools).
        const int nvalid = kKv8 ? kKeys : valid_keys(w, j);
        if (nvalid < kKeys) {
          uint8_t* vt = Vs + slot * Geo::kTileBytes;
          const int n16 = (kKeys - nvalid) * Geo::kHalves * 8;
          for (int i = lane; i < n16; i += 32) {
            const int row = nvalid + i / (Geo::kHalves * 8);
            const int rem = i % (Geo::kHalves * 8);
            *reinterpret_cast<U4*>(vt + (rem >> 3) * Geo::kHalfBytes + row * 128 +
                                   (rem & 7) * 16) = U4{0, 0, 0, 0};
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        // per head: O_x += P_x V_j as soon as P_x is ready, then S_x for the next tile (it
        // overwrites P_x in TMEM, so it must follow the P.V MMA, which tcgen05 keeps in order)
        const bool more = j + 1 < w.n_tiles;
        const int nslot = (it + 1) % kStagesK;
        for (int x = 0; x < hpc; ++x) {
          if (!warp_wait_bounded(&p_ready[x], it & 1, abort_flag, p.err, kErrPrefillWait)) {
            ok = false;
            break;
          }
          if (lane == 0) {
            tc_fence_after();
            issue_o(x, it, j == 0);
            if (x == hpc - 1) umma_commit(&v_empty[slot]);
          }
          __syncwarp();
          if (more) {
            if (!warp_wait_bounded(&k_in[nslot], ((it + 1) / kStagesK) & 1, abort_flag,
                                   p.err, kErrPrefillWait)) {
              ok = false;
              break;
            }
            if (lane == 0) {
              tc_fence_after();
              issue_s(x, it + 1);
              if (x == hpc - 1) {
                umma_commit(&k_empty[nslot]);
                if (j + 2 == w.n_tiles) umma_commit(q_empty);  // the unit's last S
              }
            }
            __syncwarp();
          }
        }
      }
      kv_iter += w.n_tiles;
    }
    // every MMA issued so far must finish before TMEM is released
    if (lane == 0) umma_commit(mma_done);
    __syncwarp();
    warp_wait_bounded(mma_done, 0, never, nullptr, 0, kWaitTimeoutNs / 8);
  } else if (kFuse && p.fuse_rows > 0) {
    // ------------------------------------------------------------------ KV write (warps 2-3)
    // For each unit whose first query head is its KV group's first, the query tile's new K
    // and V rows of that KV head, from the first key the attention reads out of k_new / v_new,
    // are copied into their cache slots (one 16-byte chunk per thread and step).  Nothing in
    // this launch reads those slots; the older rows that share a box were written before it.
    const int wt = (warp - 2) * 32 + lane;
    constexpr int kChunks = D / 8;  // 16-byte chunks per row
    for (int k = 0;; ++k) {
      const int u = unit_index(k);
      if (u >= num_units) break;
      const int tile_idx = u / groups;
      const int hq0 = (u - tile_idx * groups) * hpc;
      if (hq0 % G != 0) continue;
      const PrefillTile tile = p.tiles ? p.tiles[tile_idx] : inl.v[tile_idx];
      const int h = hq0 / G;
      const int past = tile.kv_len - tile.q_len;
      const int edge = (past + p.fuse_rows - 1) / p.fuse_rows * p.fuse_rows;
      const int i0 = max(tile.q_start, edge - past);  // local token indices [i0, i1)
      const int i1 = min(tile.q_len, tile.q_start + kRows);
      const int rows = i1 - i0;
      if (rows <= 0) continue;
      const int32_t* bt_row =
          p.kv.layout == 0 ? p.kv.block_table + (size_t)tile.seq * p.kv.max_blocks
                           : p.kv.block_table +
                                 ((size_t)tile.seq * p.kv.num_kv_heads + h) * p.kv.max_blocks;
      // four 16-byte loads in flight per thread before their stores
      const int total = 2 * rows * kChunks;
      for (int c0 = wt; c0 < total; c0 += 64 * 4) {
        uint4 val[4];
        uint4* dst[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int c = c0 + q * 64;
          dst[q] = nullptr;
          if (c >= total) continue;
          const int kvsel = c / (rows * kChunks);
          const int rem = c - kvsel * rows * kChunks;
          const int i = i0 + rem / kChunks;
          const int ch = rem % kChunks;
          const int pos = past + i;
          const int blk = pos >> log2P;
          const int page = blk < p.kv.max_blocks ? __ldg(bt_row + blk) : -1;
          if (page < 0 || page >= p.kv.num_pages) {
            atomicOr(p.err, kErrBadIndex);
            continue;
          }
          const int slot = pos & (P - 1);
          const size_t row = p.kv.layout == 0
                                 ? ((size_t)page * P + slot) * p.kv.num_kv_heads + h
                                 : (size_t)page * P + slot;
          val[q] = __ldg(reinterpret_cast<const uint4*>(
                             (kvsel == 0 ? p.k_new : p.v_new) +
                             ((size_t)(tile.t0 + i) * p.kv.num_kv_heads + h) * D) +
                         ch);
          dst[q] = reinterpret_cast<uint4*>(
                       static_cast<uint16_t*>(kvsel == 0 ? p.k_pool_w : p.v_pool_w) + row * D) +
                   ch;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (dst[q]) __stcs(dst[q], val[q]);  // streaming: nothing here reads them again
      }
    }
  } else if (kKv8) {
    // ------------------------------------------------------------------ e4m3 -> f16 (warps 2-3)
    // Each unit's Q tiles are converted in place (bf16 -> f16, position for position); each
    // K and V tile's codes, which the TMA put in the upper half of the slot (row r's 128 codes
    // in the 128-byte line of row r, 16-byte chunk c at chunk c ^ (r & 7), the 128-byte
    // swizzle), are expanded into both halves of the slot in the layout a bf16 tile has.  A
    // thread does whole rows: the upper half of row r is written only after all its codes were
    // read (dims 0..63 go to the lower half first), so the expansion is in place.  V rows past
    // the tile's last real key are written as zeros.
    const int wt = (warp - 2) * 32 + lane;
    // rows wt and wt + 64 of a tile (same swizzle phase), one 16-byte chunk of each per step
    auto expand_rows = [&](uint8_t* t, bool valid0, bool valid1) {
      uint8_t* line0 = t + wt * 128;
      uint8_t* line1 = t + Geo::kHalfBytes + wt * 128;
      const int sw = wt & 7;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {  // codes of dims 16c .. 16c + 15
        const int ic = (c ^ sw) << 4;
        const U4 in0 = valid0 ? *reinterpret_cast<const U4*>(line1 + ic) : U4{0u, 0u, 0u, 0u};
        const U4 in1 =
            valid1 ? *reinterpret_cast<const U4*>(line1 + 64 * 128 + ic) : U4{0u, 0u, 0u, 0u};
        uint8_t* out = c < 4 ? line0 : line1;
        const int oc = 2 * (c & 3);  // chunk of dims 16c .. 16c + 7 within its half
        const int o0 = (oc ^ sw) << 4, o1 = ((oc + 1) ^ sw) << 4;
        *reinterpret_cast<U4*>(out + o0) =
            U4{e4m3x2_to_f16x2(in0.x), e4m3x2_to_f16x2(in0.x >> 16), e4m3x2_to_f16x2(in0.y),
               e4m3x2_to_f16x2(in0.y >> 16)};
        *reinterpret_cast<U4*>(out + o1) =
            U4{e4m3x2_to_f16x2(in0.z), e4m3x2_to_f16x2(in0.z >> 16), e4m3x2_to_f16x2(in0.w),
               e4m3x2_to_f16x2(in0.w >> 16)};
        *reinterpret_cast<U4*>(out + 64 * 128 + o0) =
            U4{e4m3x2_to_f16x2(in1.x), e4m3x2_to_f16x2(in1.x >> 16), e4m3x2_to_f16x2(in1.y),
               e4m3x2_to_f16x2(in1.y >> 16)};
        *reinterpret_cast<U4*>(out + 64 * 128 + o1) =
            U4{e4m3x2_to_f16x2(in1.z), e4m3x2_to_f16x2(in1.z >> 16), e4m3x2_to_f16x2(in1.w),
               e4m3x2_to_f16x2(in1.w >> 16)};
      }
    };
    bool ok = true;
    int kv_iter = 0;  // K/V tiles converted, over all units of this CTA
    int q_iter = 0;   // units with key tiles
    for (int k = 0; ok; ++k) {
      const int u = unit_index(k);
      if (u >= num_units) break;
      const Unit w = unit_at(u);
      if (w.n_tiles == 0) continue;
      ok = warp_wait_bounded(q_full, q_iter & 1, abort_flag, p.err, kErrPrefillWait);
      ++q_iter;
      if (!ok) break;
      for (int i = wt; i < hpc * Geo::kTileBytes / 16; i += 64) {
        U4* c = reinterpret_cast<U4*>(Qs) + i;
        U4 v = *c;
        v.x = bf16x2_to_f16x2(v.x);
        v.y = bf16x2_to_f16x2(v.y);
        v.z = bf16x2_to_f16x2(v.z);
        v.w = bf16x2_to_f16x2(v.w);
        *c = v;
      }
      fence_proxy_async_smem();  // the tensor cores read these through the async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive(q_conv);
      for (int j = 0; ok && j < w.n_tiles; ++j) {
        const int it = kv_iter + j;
        const int nvalid = valid_keys(w, j);
        for (int kv = 0; kv < 2; ++kv) {
          const int ns = kv == 0 ? kStagesK : kStagesV;
          const int slot = it % ns;
          if (!warp_wait_bounded(kv == 0 ? &k_full[slot] : &v_full[slot], (it / ns) & 1,
                                 abort_flag, p.err, kErrPrefillWait)) {
            ok = false;
            break;
          }
          uint8_t* t = (kv == 0 ? Ks : Vs) + slot * Geo::kTileBytes;
          expand_rows(t, kv == 0 || wt < nvalid, kv == 0 || wt + 64 < nvalid);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(kv == 0 ? &k_conv[slot] : &v_conv[slot]);
        }
      }
      kv_iter += w.n_tiles;
    }
  }
  } else if ((warp - 4) / 4 < hpc) {
    // ------------------------------------------------------------------ softmax (head x)
    regs_alloc<kRegsSoftmax>();
    const int x = (warp - 4) / 4;
    const int wq = warp & 3;                        // TMEM lane quarter of this warp
    const int r = wq * 32 + lane;                   // query row == TMEM lane
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t ts = tmem + x * 128 + lane_off;
    const uint32_t to = tmem + 256 + x * 128 + lane_off;
    bool ok = true;
    int it0 = 0;  // S tiles of this head before the current unit
    for (int k = 0; ok; ++k) {
      const int u = unit_index(k);
      if (u >= num_units) break;
      const Unit w = unit_at(u);
      const PrefillTile& tile = w.tile;
      const int32_t* table = w.table;
      const int n_entries = w.n_entries;
      const int n_tiles = w.n_tiles;
      const int past = w.past;
      const int h = w.h;
      const int hq = w.hq0 + x;
      const int q_local = tile.q_start + r;
      const int pos = past + q_local;                 // absolute position of this row
      const int lim = p.causal ? min(tile.kv_len, pos + 1) : tile.kv_len;
      const float sc = p.k_scale ? p.scale_log2 * __ldg(p.k_scale + h) : p.scale_log2;
      float m_ref = -CUDART_INF_F, l = 0.f;
      for (int j = 0; j < n_tiles; ++j) {
        if (!warp_wait_bounded(&s_full[x], (it0 + j) & 1, abort_flag, p.err,
                               kErrPrefillWait)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sr[kKeys];
#pragma unroll
        for (int c = 0; c < kKeys / 32; ++c) tmem_ld32(ts + c * 32, sr + c * 32);
        // first key position of each column group: dense -> j*128; sparse -> lane e holds the
        // start of the tile's e-th table block (missing entries map past every limit)
        int ent = j * kKeys;
        int tile_last;  // last key position the tile may hold
        bool partial = false;
        if (table) {
          const int per = kKeys >> log2P;
          const int e0 = j * per;
          const int ne = min(per, n_entries - e0);
          ent = 0x3fff0000;
          if (lane < ne) ent = __ldg(table + e0 + lane) << log2P;
          tile_last = __shfl_sync(0xffffffffu, ent, ne - 1) + P - 1;
          partial = ne < per;
        } else {
          tile_last = j * kKeys + kKeys - 1;
        }
        const bool need_mask = partial || tile_last >= tile.kv_len ||
                               (p.causal && tile_last > past + tile.q_start);
        tmem_wait_ld();
        uint32_t vis[kKeys / 32];  // visibility bits (masked tiles only)
        if (need_mask) {
#pragma unroll
          for (int w = 0; w < kKeys / 32; ++w) vis[w] = 0u;
#pragma unroll
          for (int c = 0; c < kKeys; ++c) {
            const int kp = table ? __shfl_sync(0xffffffffu, ent, c >> log2P) + (c & (P - 1))
                                 : ent + c;
            vis[c >> 5] |= (kp < lim ? 1u : 0u) << (c & 31);
          }
        }
        // The reference max m_ref comes from the first tile in which the row sees a key; later
        // tiles take P against it with no max pass, so P may exceed 1.  That costs no precision
        // (fp32 and bf16 are relative formats) until a tile's row sum passes 2^64; such a tile,
        // rare in practice, is redone once against its own max, with O and l rescaled.
        bool need_max = m_ref == -CUDART_INF_F;
        float fac = 1.f;
        bool rescale = false;
        float rs;
#pragma unroll 1
        for (int attempt = 0;; ++attempt) {
          if (__any_sync(0xffffffffu, need_max)) {
            // row max of scale*S over the visible columns: short trees of independent
            // accumulators, not a 128-long dependency chain
            float mx;
            if (need_mask) {
              float acc[8];
#pragma unroll
              for (int k = 0; k < 8; ++k) acc[k] = -CUDART_INF_F;
#pragma unroll
              for (int c = 0; c < kKeys; ++c)
                acc[c & 7] = fmaxf(acc[c & 7], (vis[c >> 5] >> (c & 31)) & 1u
                                                   ? __uint_as_float(sr[c]) * sc
                                                   : -CUDART_INF_F);
              mx = fmaxf(fmaxf(fmaxf(acc[0], acc[1]), fmaxf(acc[2], acc[3])),
                         fmaxf(fmaxf(acc[4], acc[5]), fmaxf(acc[6], acc[7])));
            } else {
              // scale*max(S) for a non-negative scale, scale*min(S) for a negative one;
              // 3-input max/min: two new values per instruction, four accumulators
              float acc[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) acc[k] = __uint_as_float(sr[k]);
              if (sc >= 0.f) {
#pragma unroll
                for (int c = 4; c < kKeys; c += 2)
                  acc[(c >> 1) & 3] = fmax3(acc[(c >> 1) & 3], __uint_as_float(sr[c]),
                                            __uint_as_float(sr[c + 1]));
                mx = fmaxf(fmax3(acc[0], acc[1], acc[2]), acc[3]) * sc;
              } else {
#pragma unroll
                for (int c = 4; c < kKeys; c += 2)
                  acc[(c >> 1) & 3] = fmin3(acc[(c >> 1) & 3], __uint_as_float(sr[c]),
                                            __uint_as_float(sr[c + 1]));
                mx = fminf(fmin3(acc[0], acc[1], acc[2]), acc[3]) * sc;
              }
            }
            if (need_max && mx > m_ref) {  // mx = -inf: still no visible key
              if (m_ref != -CUDART_INF_F) {
                fac = fast_exp2(m_ref - mx);
                rescale = true;
              }
              m_ref = mx;
            }
          }
          const float neg_m = m_ref == -CUDART_INF_F ? 0.f : -m_ref;
          // P = exp2(scale*S - m): one packed FFMA per pair of elements and one EX2 per
          // element; the row sum is kept in four packed partial sums.  The loop exists twice:
          // most tiles see every key and take the version without the visibility selects.
          const uint64_t sc2 = f2_pack(sc, sc);
          const uint64_t nm2 = f2_pack(neg_m, neg_m);
          uint64_t rsum2[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) rsum2[k] = 0ull;
          auto exp_pass = [&](auto masked) {
            constexpr bool kMasked = decltype(masked)::value;
#pragma unroll
            for (int c = 0; c < kKeys; c += 2) {
              float t0, t1;
              f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sc2,
                               nm2),
                        t0, t1);
              float p0 = fast_exp2(t0);
              float p1 = fast_exp2(t1);
              if constexpr (kMasked) {
                p0 = (vis[c >> 5] >> (c & 31)) & 1u ? p0 : 0.f;
                p1 = (vis[(c + 1) >> 5] >> ((c + 1) & 31)) & 1u ? p1 : 0.f;
              }
              rsum2[(c >> 1) & 3] = f2_add(rsum2[(c >> 1) & 3], f2_pack(p0, p1));
              // P as bf16 (f16 for e4m3 pools) pairs, over the consumed S values
              sr[c >> 1] = kKv8 ? pack_f16(p0, p1) : pack_bf16(p0, p1);
            }
          };
          if (need_mask)
            exp_pass(std::true_type{});
          else
            exp_pass(std::false_type{});
          rs = 0.f;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            float a, b;
            f2_unpack(rsum2[k], a, b);
            rs += a + b;
          }
          const bool over = !(rs <= (kKv8 ? kMaxTileSumF16 : kMaxTileSum));
          if (attempt > 0 || !__any_sync(0xffffffffu, over)) break;
          need_max = over;
#pragma unroll
          for (int c = 0; c < kKeys / 32; ++c) tmem_ld32(ts + c * 32, sr + c * 32);
          tmem_wait_ld();
        }
        l = l * fac + rs;
#pragma unroll
        for (int c = 0; c < kKeys / 64; ++c) tmem_st32(ts + c * 32, sr + c * 32);
        if (j > 0 && __any_sync(0xffffffffu, rescale)) {
          // O += P V of the previous tile must be complete before O is rescaled
          if (!warp_wait_bounded(&o_done[x], (it0 + j - 1) & 1, abort_flag, p.err,
                                 kErrPrefillWait)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(to + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * fac);
            tmem_st32(to + c * 32, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_ready[x]);
      }
      // ---- epilogue: O / l -> bf16 (a row that saw no key gets 0 and lse = -inf)
      if (ok && n_tiles > 0) {
        ok = warp_wait_bounded(&o_done[x], (it0 + n_tiles - 1) & 1, abort_flag, p.err,
                               kErrPrefillWait);
        tc_fence_after();
      }
      if (ok) {
        const int t = tile.t0 + q_local;
        const bool write = q_local < tile.q_len;
        uint16_t* orow = p.out + ((size_t)t * Hq + hq) * D;
        const float inv = l > 0.f ? (p.v_scale ? __ldg(p.v_scale + h) : 1.f) / l : 0.f;
        // a thread writes its own row: each store instruction of the warp touches 32 rows, so
        // the widest store (32 bytes, when the output is 32-byte aligned) halves the count
        const bool wide = (reinterpret_cast<uintptr_t>(p.out) & 31) == 0;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          if (n_tiles > 0) {
            tmem_ld32(to + c * 32, o);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = 0u;
          }
          if (write) {
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              w[i] = pack_bf16(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
            if (wide) {
              st_global_v8(orow + c * 32, w);
              st_global_v8(orow + c * 32 + 16, w + 8);
            } else {
#pragma unroll
              for (int i = 0; i < 16; i += 4)
                *reinterpret_cast<U4*>(orow + c * 32 + 2 * i) = U4{w[i], w[i + 1], w[i + 2], w[i + 3]};
            }
          }
        }
        if (write && p.lse)
          p.lse[(size_t)t * Hq + hq] =
              l > 0.f ? (m_ref + fast_log2(l)) * 0.69314718055994531f : -CUDART_INF_F;
      }
      it0 += n_tiles;
    }
  } else {
    regs_dealloc<kRegsControl>();  // head B's warpgroup when the group size is odd
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

template <int D, bool kFuse, bool kKv8>
cudaError_t launch_prefill_kernel(const CUtensorMap& qmap, const CUtensorMap& kmap,
                                  const CUtensorMap& vmap, const CUtensorMap& knmap,
                                  const CUtensorMap& vnmap, const PrefillLaunch& p,
                                  const PrefillTilesInline* inl, dim3 grid, cudaStream_t stream) {
  const void* k = reinterpret_cast<const void*>(prefill_kernel<D, kFuse, kKv8>);
  // the register rebalancing inside the kernel needs exactly the launch budget it was
  // written for; refuse to launch otherwise (a short budget would stall setmaxnreg.inc)
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, k);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) {
    set_last_error("prefill kernel built with %d registers per thread, expected %d", fa.numRegs,
                   kLaunchRegs);
    return cudaErrorInvalidConfiguration;
  }
  e = ensure_smem_attr(k, PfGeom<D>::kAlloc);
  if (e != cudaSuccess) return e;
  if (!p.launched) {
    prefill_kernel<D, kFuse, kKv8><<<grid, kThreads, PfGeom<D>::kAlloc, stream>>>(
        qmap, kmap, vmap, knmap, vnmap, p, *inl);
    return cudaSuccess;
  }
  // the event fires once every CTA has started: work that waits for it on another stream
  // gets only the SMs these CTAs left
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = PfGeom<D>::kAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeLaunchCompletionEvent;
  attr[0].val.launchCompletionEvent.event = p.launched;
  attr[0].val.launchCompletionEvent.flags = 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, prefill_kernel<D, kFuse, kKv8>, qmap, kmap, vmap, knmap, vnmap,
                            p, *inl);
}

cudaError_t launch_prefill(const PrefillLaunch& p, const PrefillTilesInline* inl,
                           cudaStream_t stream) {
  if (p.num_tiles <= 0) return cudaSuccess;
  CUtensorMap qmap, kmap, vmap;
  cudaError_t e = encode_q_map(&qmap, p.q, p.num_tokens, p.num_q_heads, p.head_dim, kRows);
  if (e != cudaSuccess) return e;
  e = encode_kv_map(&kmap, p.kv.k_pool, p.kv, p.head_dim, kKeys);
  if (e != cudaSuccess) return e;
  e = encode_kv_map(&vmap, p.kv.v_pool, p.kv, p.head_dim, kKeys);
  if (e != cudaSuccess) return e;
  // this step's new rows [T, Hkv, D], in boxes as high as the pool's
  CUtensorMap knmap = kmap, vnmap = vmap;
  if (p.fuse_rows > 0) {
    e = encode_q_map(&knmap, p.k_new, p.num_tokens, p.num_kv_heads, p.head_dim, p.fuse_rows);
    if (e != cudaSuccess) return e;
    e = encode_q_map(&vnmap, p.v_new, p.num_tokens, p.num_kv_heads, p.head_dim, p.fuse_rows);
    if (e != cudaSuccess) return e;
  }
  const int G = p.num_q_heads / p.num_kv_heads;
  const int hpc = (p.qtile_table == nullptr && (G & 1) == 0) ? 2 : 1;  // as in the kernel
  // persistent: one CTA per SM at most (each holds all of an SM's TMEM); otherwise one CTA
  // per unit, which the kernel's unit walk reduces to its first unit
  const long units = (long)p.num_tiles * (p.num_q_heads / hpc);
  long ctas = units;
  if (p.persistent) {
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if (ctas > sms) ctas = sms;
    if (p.max_ctas > 0 && ctas > p.max_ctas) ctas = p.max_ctas;
  }
  const dim3 grid((unsigned)ctas);
  const bool fuse = p.fuse_rows > 0;
  if (p.kv.kv8) {
    // e4m3 pools: codes converted inside the kernel (head_dim 128, no fused write)
    if (p.head_dim != 128 || fuse || !p.k_scale || !p.v_scale) {
      set_last_error("e4m3 pools on the tensor-core kernel need head_dim 128, both scale "
                     "vectors and no fused write");
      return cudaErrorInvalidValue;
    }
    e = launch_prefill_kernel<128, false, true>(qmap, kmap, vmap, knmap, vnmap, p, inl, grid,
                                                stream);
  } else if (p.head_dim == 128) {
    e = fuse ? launch_prefill_kernel<128, true, false>(qmap, kmap, vmap, knmap, vnmap, p, inl,
                                                       grid, stream)
             : launch_prefill_kernel<128, false, false>(qmap, kmap, vmap, knmap, vnmap, p, inl,
                                                        grid, stream);
  } else {
    e = fuse ? launch_prefill_kernel<64, true, false>(qmap, kmap, vmap, knmap, vnmap, p, inl,
                                                      grid, stream)
             : launch_prefill_kernel<64, false, false>(qmap, kmap, vmap, knmap, vnmap, p, inl,
                                                       grid, stream);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace rpa
