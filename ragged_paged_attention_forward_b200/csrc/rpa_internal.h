// Internal declarations shared by the host planner (rpa_api.cpp) and the kernels (*.cu).
// Nothing here is part of the public ABI (include/rpa.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace rpa {

// Keys handled by one pipeline stage of the decode kernel and by one tensor-core tile of the
// prefill kernel.
constexpr int kDecodeStageKeys = 64;
constexpr int kPrefillTileKeys = 128;
constexpr int kPrefillTileRows = 128;
constexpr int kMaxSparsePage = 128;  // block-union tables: largest page (= table block) size
constexpr int kMaxSplitKeys = 4096;
constexpr int kMinSplitKeys = 256;

// Work lists of up to kInlineItems entries travel as kernel parameters (no host-to-device
// copy); longer lists go through the workspace.
constexpr int kInlineItems = 256;

// Device error word codes (OR-ed together).
enum DeviceErrorCode : int {
  kErrDecodeWait = 1 << 0,
  kErrPrefillWait = 1 << 1,
  kErrBadIndex = 1 << 2,
  kErrBadPosition = 1 << 3,
  kErrLimits = 1 << 4,       // a device-planned step exceeded the plan's limits
};

// One (sequence, key range) item of the split-KV decode kernel; one CTA per (item, KV head).
struct DecodeItem {
  int32_t seq;
  int32_t t0;         // first query token of the sequence
  int32_t q_len;      // query tokens (all of them: a decode item covers the whole query)
  int32_t kv_len;
  int32_t k_begin;    // key range [k_begin, k_end), k_begin a multiple of kDecodeStageKeys
  int32_t k_end;
  int32_t part_slot;  // -1: single split, write the final output; else partial-result slot
  int32_t pad;
};
static_assert(sizeof(DecodeItem) == 32, "DecodeItem layout");

// One query token whose decode splits are merged (log-sum-exp reduce).
struct MergeRow {
  int32_t token;
  int32_t local;       // query index inside its sequence
  int32_t first_slot;  // partial slots first_slot .. first_slot + nsplit - 1
  int32_t nsplit;
};
static_assert(sizeof(MergeRow) == 16, "MergeRow layout");

// One 128-query-token tile of the prefill kernel; one CTA per (tile, query head).
struct PrefillTile {
  int32_t seq;
  int32_t t0;       // first query token of the sequence
  int32_t q_len;
  int32_t kv_len;
  int32_t q_start;  // local index of the tile's first query
  int32_t pad[3];
};
static_assert(sizeof(PrefillTile) == 32, "PrefillTile layout");

struct DecodeItemsInline {
  DecodeItem v[kInlineItems];
};
struct MergeRowsInline {
  MergeRow v[kInlineItems];
};
struct PrefillTilesInline {
  PrefillTile v[kInlineItems];
};

struct PagedKV {
  const void* k_pool;
  const void* v_pool;
  const int32_t* block_table;
  int32_t layout;          // 0 seq-major, 1 head-major
  int32_t page_size;
  int32_t log2_page;
  int32_t max_blocks;
  int32_t num_kv_heads;
  int32_t num_pages;
  int32_t kv8;             // 1: the pools hold e4m3 codes (one byte per element)
};

struct DecodeLaunch {
  const DecodeItem* items;   // null: the items are the kernel's inline parameter list
  int32_t num_items;
  const int32_t* count;      // device-planned steps: number of valid items (null: num_items)
  int32_t rows_per_item;     // 8 * NT: stride of the partial-result rows
  const uint16_t* q;         // bf16 [T, Hq, D]
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t causal;
  float scale_log2;          // softmax scale * log2(e)
  uint16_t* out;             // bf16 [T, Hq, D]
  float* lse;                // [T, Hq] or null
  float* part_o;             // [slots, Hkv, rows_per_item, D]
  float* part_lse;           // [slots, Hkv, rows_per_item] (log2 domain)
  int* err;
  PagedKV kv;
  // KV write fused into the decode kernel (pure decode batches): each CTA first writes the
  // new tokens whose positions fall in its key range, for its KV head.  Null: no write.
  const uint16_t* k_new;     // bf16 [T, Hkv, D]
  const uint16_t* v_new;
  void* k_pool_w;            // bf16 pools, or e4m3 code pools when kv.kv8
  void* v_pool_w;
  // e4m3 pools (kv.kv8): element = code * scale[kv head]; new tokens are stored as
  // e4m3(fp32(x) / scale), nearest even, saturating
  const float* k_scale;      // [Hkv]
  const float* v_scale;      // [Hkv]
  // diagnostics (tests of the bounded waits): nonzero = load no K/V and give up every wait
  // after this many nanoseconds, so the waits run out and the kernel reports it
  uint32_t test_wait_ns;
};

struct MergeLaunch {
  const MergeRow* rows;      // null: inline parameter list
  int32_t num_rows;
  const int32_t* count;      // device-planned steps: number of valid rows (null: num_rows)
  int32_t rows_per_item;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  const float* part_o;
  const float* part_lse;
  uint16_t* out;
  float* lse;
};

struct PrefillLaunch {
  const PrefillTile* tiles;  // null: inline parameter list
  int32_t num_tiles;
  const int32_t* count;      // device-planned steps: number of valid tiles (null: num_tiles)
  const uint16_t* q;
  int32_t num_tokens;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t causal;
  float scale_log2;
  uint16_t* out;
  float* lse;
  const int32_t* group_table;  // [B, Hkv, max_blocks] or null
  const int32_t* group_count;  // [B, Hkv] or null
  // per-(query tile, query head) tables instead (block-sparse execution, one head per CTA):
  // [B, Hq, qtiles_per_seq, max_blocks] and [B, Hq, qtiles_per_seq], or null
  const int32_t* qtile_table;
  const int32_t* qtile_count;
  int32_t qtiles_per_seq;
  // per-KV-head factors on the scores and the output (the e4m3 path reads exact bf16 copies
  // of the codes: K = code * k_scale[h], V = code * v_scale[h]); null: 1
  const float* k_scale;
  const float* v_scale;
  // 1: one CTA per SM walks the units (a launch that has the GPU to itself); 0: one CTA per
  // unit, so that a decode kernel running beside it takes SMs as units finish
  int32_t persistent;
  // persistent launches: at most this many CTAs (0: one per SM), and, when set, an event
  // recorded once every CTA of the launch has started (host-side fields)
  int32_t max_ctas;
  cudaEvent_t launched;
  int* err;
  PagedKV kv;
  // KV write fused into this kernel (bf16 pools): when fuse_rows > 0, a TMA box of keys that
  // starts at or past round_up(past, fuse_rows) -- fuse_rows is the box height, min(P, 128)
  // -- is read from this step's k_new / v_new rows instead of the pool, and the unit of each
  // (query tile, KV head) whose first query head is the group's first copies the tile's new
  // rows from that boundary on into the pool.  New rows that share a box with older keys
  // are written before the launch.  0: every key from the pool, nothing written.
  const uint16_t* k_new;     // bf16 [T, Hkv, D]
  const uint16_t* v_new;
  void* k_pool_w;
  void* v_pool_w;
  int32_t fuse_rows;
};

struct WriteLaunch {
  const uint16_t* k_new;
  const uint16_t* v_new;
  void* k_pool;              // bf16 pools, or e4m3 code pools when kv8
  void* v_pool;
  int32_t kv8;               // 1: store e4m3(fp32(x) / scale[kv head]) codes
  const float* k_scale;      // [Hkv] (kv8)
  const float* v_scale;
  const int32_t* block_table;
  const int32_t* cu_seqlens_q;
  const int32_t* seq_lens_k;
  int32_t num_seqs;
  int32_t num_tokens;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t page_size;
  int32_t max_blocks;
  int32_t layout;
  int32_t num_pages;
  int32_t tokens_on_device;  // 1: num_tokens is a bound, the step has cu_seqlens_q[num_seqs]
  // > 0: skip the tokens of sequences with q_len * group <= skip_rows_upto (their rows go to
  // the decode kernel, which writes them itself)
  int32_t skip_rows_upto;
  int32_t group;
  // > 0: only positions below round_up(past, below_box) -- the new rows that share a TMA box
  // with older keys, which the tensor-core kernel reads from the pool
  int32_t below_box;
  int* err;
};

struct RotaryLaunch {
  const uint16_t* q;      // [T, Hq, D] or packed [T, (Hq + 2 Hkv) D]
  const uint16_t* k;      // [T, Hkv, D] or null (packed)
  const uint16_t* v;
  const uint16_t* cos;    // [max_pos, rd/2] or null (no rotation)
  const uint16_t* sin;
  int32_t max_pos;
  int32_t rotary_dim;
  int32_t interleaved;
  uint16_t* q_out;        // [T, Hq, D]
  uint16_t* k_pool;
  uint16_t* v_pool;
  const int32_t* block_table;
  const int32_t* cu_seqlens_q;
  const int32_t* seq_lens_k;
  int32_t num_seqs;
  int32_t num_tokens;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t page_size;
  int32_t max_blocks;
  int32_t layout;
  int32_t num_pages;
  int* err;
};

// The device-side planner: reads the step's lengths on the device and writes the work lists
// (and their sizes) into the workspace, so that a step needs no host arrays and can be
// captured in a CUDA graph.  Limits are fixed when the plan is made.
struct PlanDeviceLaunch {
  const int32_t* cu_seqlens_q;   // [B+1]
  const int32_t* seq_lens_k;     // [B]
  int32_t num_seqs;
  int32_t max_tokens;
  int32_t max_kv_len;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t causal;
  int32_t split_keys;
  int32_t decode_rows;           // a sequence goes to the decode kernel when q_len * G <= this
  int32_t cap_items, cap_rows, cap_tiles;
  DecodeItem* items;
  MergeRow* rows;
  PrefillTile* tiles;
  int32_t* counts;               // [3]: items, merge rows, tiles
  int* err;
};

// Launchers (return the cudaError_t of the launch).
cudaError_t launch_write_kv(const WriteLaunch& p, cudaStream_t stream);
cudaError_t launch_plan_device(const PlanDeviceLaunch& p, cudaStream_t stream);
cudaError_t launch_rotary_write(const RotaryLaunch& p, cudaStream_t stream);
cudaError_t launch_decode(const DecodeLaunch& p, const DecodeItemsInline* inl, int nt,
                          cudaStream_t stream);
cudaError_t launch_merge(const MergeLaunch& p, const MergeRowsInline* inl, cudaStream_t stream);
cudaError_t launch_prefill(const PrefillLaunch& p, const PrefillTilesInline* inl,
                           cudaStream_t stream);
cudaError_t launch_qtile_tables(const uint8_t* mask, int B, int Hq, int nqb, int nkb,
                                int qb_per_tile, int ntiles, int32_t* table, int32_t* count,
                                cudaStream_t stream);
cudaError_t launch_group_tables(const uint8_t* mask, int B, int Hq, int Hkv, int nqb, int nkb,
                                int32_t* table, int32_t* count, cudaStream_t stream);

// Device error word of the current device (allocated by the library, lives until exit).
cudaError_t device_error_word(int** ptr);

// Host helpers (launch_util.cpp).
// TMA map over a K or V pool seen as 4-D (dims, kv heads, slots, pages), innermost first; the
// head-major pool is the same with a single "head".  Box: 64 dims x 1 head x
// min(page_size, box_keys) slots x 1 page, 128-byte swizzle.
cudaError_t encode_kv_map(CUtensorMap* map, const void* pool, const PagedKV& kv, int head_dim,
                          int box_keys);
// TMA map over Q [T, Hq, D] seen as 3-D (dims, heads, tokens); box 64 x 1 x box_rows.
cudaError_t encode_q_map(CUtensorMap* map, const void* q, int num_tokens, int num_q_heads,
                         int head_dim, int box_rows);
// Raise a kernel's dynamic shared-memory limit once per device.
cudaError_t ensure_smem_attr(const void* kernel, int bytes);
// A non-blocking stream of the current device owned by the library (created once), on which
// the tensor-core kernel of a mixed batch runs next to the split-KV decode kernel.
cudaError_t side_stream(cudaStream_t caller, cudaStream_t* stream);
int device_sm_count();

// Sets the thread-local error text returned by rpa_last_error().
void set_last_error(const char* fmt, ...);

}  // namespace rpa
