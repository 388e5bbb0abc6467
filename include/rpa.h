/*
 * rpa.h -- ragged paged attention for NVIDIA B200 (sm_100a): the C ABI of librpa.so.
 *
 * One call attends a packed, variable-length batch of query tokens from many sequences
 * (pure decode, pure prefill, or a mix) against a KV cache held in fixed-size pages that
 * each sequence reaches through a block table, and writes the new tokens' K/V into their
 * cache slots first.  The method is the one of "Ragged Paged Attention: A High-Performance
 * and Flexible LLM Inference Kernel for TPU" (Key ideas: ragged tiling over paged KV, the
 * cache write fused with attention, specialised decode / prefill / mixed kernels); the
 * operator's inputs and conventions follow "[WebGPU] Optimized PagedAttention
 * implementation (2/n)" (packed varlen Q with cumulative_seqlens_q, seqlens_k, block_table,
 * a paged cache of shape (num_blocks, block_size, kv_num_heads, head_size), in-place cache,
 * token_count == 0 is a no-op); the per-group block tables and the KV-head-major layout
 * follow "CompactAttention: Accelerating Chunked Prefill with Block-Union KV Selection"
 * (Core claim; Fig. 3; Fig. 4).
 *
 * Notation: B sequences, T = cu_seqlens_q[B] query tokens, Hq query heads, Hkv KV heads
 * (Hq % Hkv == 0, G = Hq / Hkv, query head hq reads KV head hq / G), head dim D, page size P.
 * q_len_b = cu_seqlens_q[b+1] - cu_seqlens_q[b]; kv_len_b = seq_lens_k[b] is the context
 * length INCLUDING the q_len_b new tokens, which occupy positions past_b .. kv_len_b - 1
 * with past_b = kv_len_b - q_len_b.  Query i of sequence b sits at position past_b + i and,
 * when causal, sees keys 0 .. past_b + i.
 *
 * Memory: every device buffer, the workspace and the stream belong to the caller.  All
 * bf16 tensors are dense row-major with the shapes given; every device pointer must be
 * 16-byte aligned.  Calls are asynchronous on the given stream (a cudaStream_t passed as
 * void*; NULL = the legacy default stream); argument errors are detected on the host,
 * returned at once, and nothing is launched.  Functions are thread-safe except that a
 * plan must not be used by two threads at once.
 */
#ifndef RPA_H
#define RPA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RPA_API __attribute__((visibility("default")))
#else
#define RPA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum rpa_status {
  RPA_OK = 0,
  RPA_ERR_INVALID_ARG = -1,          /* null/misaligned pointer, inconsistent arguments   */
  RPA_ERR_UNSUPPORTED = -2,          /* a shape or mode this build does not implement     */
  RPA_ERR_SHAPE = -3,                /* lengths that contradict each other                */
  RPA_ERR_WORKSPACE_TOO_SMALL = -4,  /* workspace smaller than rpa_plan reported          */
  RPA_ERR_CUDA = -5,                 /* a CUDA runtime call failed (see rpa_last_error)   */
  RPA_ERR_DEVICE_CHECK = -6          /* a kernel gave up a bounded wait (rpa_device_error)*/
} rpa_status;

typedef enum rpa_layout {
  /* pool [num_pages, P, Hkv, D]; block_table [B, max_blocks_per_seq]                     */
  RPA_LAYOUT_SEQ_MAJOR = 0,
  /* pool [num_pages, P, D], one page per (sequence, KV head, block);
     block_table [B, Hkv, max_blocks_per_seq] (CompactAttention, Fig. 4)                   */
  RPA_LAYOUT_HEAD_MAJOR = 1
} rpa_layout;

typedef enum rpa_batch_class {
  RPA_CLASS_AUTO = 0,
  RPA_CLASS_DECODE = 1,   /* every sequence has q_len <= 1                                 */
  RPA_CLASS_PREFILL = 2,  /* every non-empty sequence has q_len >= 32                      */
  RPA_CLASS_MIXED = 3     /* anything else                                                 */
} rpa_batch_class;

typedef struct rpa_shape {
  int32_t num_seqs;            /* B  >= 0                                                  */
  int32_t num_tokens;          /* T  == cu_seqlens_q[B]                                    */
  int32_t num_q_heads;         /* Hq                                                       */
  int32_t num_kv_heads;        /* Hkv, Hq % Hkv == 0                                       */
  int32_t head_dim;            /* D in {64, 128}                                           */
  int32_t page_size;           /* P, power of two, 16 <= P <= 256                          */
  int32_t num_pages;           /* pages in each of the K and V pools                       */
  int32_t max_blocks_per_seq;  /* last dimension of block_table (and of group_table)       */
  int32_t layout;              /* rpa_layout                                               */
  int32_t causal;              /* 1 = causal (bottom-right aligned), 0 = all kv_len keys   */
} rpa_shape;

typedef struct rpa_plan_options {
  int32_t force_class;         /* rpa_batch_class; AUTO lets the planner choose            */
  int32_t decode_split_keys;   /* keys per decode split, multiple of 64; 0 = automatic     */
  int32_t sparse;              /* 1: rpa_forward will be given group tables; 2: per-(query  */
                               /* tile, query head) tables (rpa_build_qtile_tables)         */
  int32_t kv_e4m3;             /* 1: the pools will hold e4m3 codes (rpa_forward_kv8); the  */
                               /* planner sizes the SM split of mixed batches for one-byte */
                               /* elements                                                 */
  int32_t wait_test_us;        /* diagnostics, for tests of the bounded waits only: > 0    */
                               /* makes the split-KV decode kernel load no K/V and give up */
                               /* each of its waits after this many microseconds (at most  */
                               /* 1000000), so rpa_forward computes no attention and sets  */
                               /* bit 1 of the device error word; 0 for real work          */
  int32_t reserved[3];         /* must be zero                                             */
} rpa_plan_options;

typedef struct rpa_plan_info {
  int32_t batch_class;         /* rpa_batch_class chosen                                   */
  int32_t num_decode_items;    /* (sequence, key split) items of the decode kernel         */
  int32_t num_prefill_tiles;   /* (sequence, 128-query tile) items of the prefill kernel   */
  int32_t num_merge_rows;      /* query tokens whose decode splits need the LSE merge      */
  int32_t launches_forward;    /* kernels rpa_forward launches when given k_new/v_new      */
  int32_t launches_write;      /* kernels rpa_write_kv launches                            */
  int32_t decode_split_keys;   /* split size used                                          */
  int32_t tensor_core_grid;    /* mixed batches: SMs given to a persistent tensor-core grid */
                               /* launched before the decode kernel (0: one CTA per unit)  */
  size_t workspace_bytes;      /* device workspace rpa_forward needs                       */
} rpa_plan_info;

typedef struct rpa_plan_s* rpa_plan_t;

/*
 * rpa_plan -- validate a batch and build its work lists on the host (the planner that
 * picks decode, prefill or mixed kernels: "Ragged Paged Attention ..." Key ideas,
 * distribution-aware compilation; the decode/prefill threshold q_len < 32 of the WebGPU
 * page, "Correctness invariants").
 *
 *   shape            host struct, read during the call only.
 *   cu_seqlens_q     HOST int32 [B+1], non-decreasing, cu[0] == 0, cu[B] == T.
 *   seq_lens_k       HOST int32 [B], q_len_b <= kv_len_b,
 *                    ceil(kv_len_b / P) <= max_blocks_per_seq.
 *   opts             optional (NULL = defaults).
 *   out_plan         receives a plan that owns host memory only; free with
 *                    rpa_plan_destroy.  The plan is valid for device copies of
 *                    cu_seqlens_q / seq_lens_k holding the same values.
 *   workspace_bytes  optional; receives the device workspace size rpa_forward needs
 *                    (256-byte aligned buffer supplied by the caller).
 * Returns RPA_OK, RPA_ERR_INVALID_ARG, RPA_ERR_SHAPE or RPA_ERR_UNSUPPORTED (head_dim not
 * 64/128, page size not a power of two in [16, 256], HEAD_MAJOR required for sparse).
 */
RPA_API rpa_status rpa_plan(const rpa_shape* shape, const int32_t* cu_seqlens_q,
                    const int32_t* seq_lens_k, const rpa_plan_options* opts,
                    rpa_plan_t* out_plan, size_t* workspace_bytes);

/*
 * rpa_plan_device -- a plan whose work lists are built on the device at every rpa_forward
 * call, from the device cu_seqlens_q / seq_lens_k of that call, so that a step takes no
 * host arrays, needs no host synchronisation and can be captured in a CUDA graph and
 * replayed with new lengths (the same pointers).  No counterpart in the pages; the
 * "graph-capturable, device-side planner" that follows the host planner above.
 *
 *   shape         num_seqs = B, the length of the lengths arrays (sequences may have
 *                 q_len 0); num_tokens = the largest T any step will have; the other fields
 *                 as for rpa_plan.
 *   max_kv_len    the largest seq_lens_k any step will have (<= max_blocks_per_seq * P).
 *   opts          optional; decode_split_keys as for rpa_plan; sparse and force_class are
 *                 not supported (RPA_ERR_UNSUPPORTED).
 *   workspace_bytes  receives the workspace size for these limits.
 * Each call of rpa_forward with this plan launches a one-CTA planner kernel (a sequence
 * goes to the split-KV decode kernel when q_len * G fits 8, 16 or 32 rows -- the smallest
 * of these that holds G -- else to the tensor-core kernel),
 * then every kernel with its largest grid; CTAs past the step's counts return at once.
 * A step beyond the limits (T, kv_len, q_len > kv_len) computes nothing and sets bit 16
 * of the device error word.  rpa_write_kv with this plan writes the step's tokens only.
 * The q, k_new, v_new, out and lse buffers given to rpa_forward hold num_tokens rows (the
 * bound): only the step's rows are read and written.
 */
RPA_API rpa_status rpa_plan_device(const rpa_shape* shape, int32_t max_kv_len,
                           const rpa_plan_options* opts, rpa_plan_t* out_plan,
                           size_t* workspace_bytes);

/* rpa_plan_get_info -- what the planner chose (host only, no device work). */
RPA_API rpa_status rpa_plan_get_info(rpa_plan_t plan, rpa_plan_info* info);

/* rpa_plan_destroy -- frees the plan's host memory; NULL is ignored. */
RPA_API void rpa_plan_destroy(rpa_plan_t plan);

/*
 * rpa_write_kv -- scatter the new tokens' K/V into their cache slots, in place
 * (ScatterKVToPagedCacheProgram of the WebGPU page, commit "Phase 1b.1": for token i of
 * sequence b, pos = past_b + i, page = block_table[b, pos / P], slot = pos % P; the
 * head-major layout uses block_table[b, h, pos / P] per KV head h).  Bytes are copied
 * unchanged; slots not addressed are not touched.
 *
 *   k_new, v_new       device bf16 [T, Hkv, D].
 *   k_pool, v_pool     device bf16 pools in shape.layout, updated in place.
 *   block_table        device int32, see rpa_layout.
 *   cu_seqlens_q       device int32 [B+1] (same values as given to rpa_plan).
 *   seq_lens_k         device int32 [B].
 *   workspace          unused by this call; may be NULL.
 * T == 0 returns RPA_OK and launches nothing.
 */
RPA_API rpa_status rpa_write_kv(rpa_plan_t plan, const void* k_new, const void* v_new,
                        void* k_pool, void* v_pool, const int32_t* block_table,
                        const int32_t* cu_seqlens_q, const int32_t* seq_lens_k,
                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * rpa_write_kv8 -- rpa_write_kv for e4m3 code pools (see rpa_forward_kv8): every new element
 * x of KV head h is stored as the e4m3 code nearest to fp32(x) / scale[h] (IEEE fp32 division,
 * ties to the even code, magnitudes past 448 saturate).  k_pool / v_pool are uint8 pools in
 * shape.layout; k_scale / v_scale device fp32 [Hkv].  head_dim must be a multiple of 16.
 * T == 0 returns RPA_OK and launches nothing.
 */
RPA_API rpa_status rpa_write_kv8(rpa_plan_t plan, const void* k_new, const void* v_new,
                                 void* k_pool, void* v_pool, const float* k_scale,
                                 const float* v_scale, const int32_t* block_table,
                                 const int32_t* cu_seqlens_q, const int32_t* seq_lens_k,
                                 void* stream);

/*
 * Rotary position embedding applied by rpa_rotary_write_kv ("[WebGPU] Optimized
 * PagedAttention implementation (2/n)", commit "Phase 1b.2": the rotary program rotates Q and
 * K before the K/V scatter, with position_id = past_b + s and dims >= rotary_dim copied
 * unchanged; interleaved or split pairing).
 *
 *   cos_cache, sin_cache  device bf16 [max_position, rotary_dim / 2]: row p holds cos and
 *                         sin of the angles of position p, one per rotated pair.
 *   max_position          rows of the caches; every position must be below it.
 *   rotary_dim            rotated dims per head: a multiple of 16, <= head_dim.
 *   interleaved           1: pair j is (x[2j], x[2j+1]); 0: pair j is (x[j], x[j + rd/2]).
 * Pair j of a row at position p becomes (x1 c - x2 s, x1 s + x2 c) with c = cos[p, j],
 * s = sin[p, j]; arithmetic in fp32, results rounded to bf16 (nearest even).
 */
typedef struct rpa_rotary {
  const void* cos_cache;
  const void* sin_cache;
  int32_t max_position;
  int32_t rotary_dim;
  int32_t interleaved;
  int32_t reserved;            /* must be zero */
} rpa_rotary;

/*
 * rpa_rotary_write_kv -- the step's input pass: take the new tokens' Q, K and V (separate, or
 * packed per token as [Q | K | V] columns: "... (2/n)", packed-QKV commit), rotate Q and K
 * by their positions (optional), write the queries to q_out and scatter K and V into their
 * cache slots (rpa_write_kv's index rule).  rpa_forward then runs on q_out with
 * k_new = v_new = NULL.  This pass is not in the pages' fused step; it is the "next" row
 * that folds rotary and the packed-QKV split into the KV write.
 *
 *   q            device bf16 [T, Hq, D]; or, with k == v == NULL, the packed input
 *                [T, (Hq + 2 Hkv) * D] (columns [0, Hq D) = Q, then K, then V).
 *   k, v         device bf16 [T, Hkv, D], or both NULL (packed input).
 *   rotary       host struct, read during the call; NULL = no rotation (a copy / split).
 *   q_out        device bf16 [T, Hq, D]; must not overlap q.
 *   k_pool, v_pool, block_table, cu_seqlens_q, seq_lens_k   as for rpa_write_kv.
 * Pointers 16-byte aligned.  T == 0 returns RPA_OK and launches nothing.  Positions at or
 * past max_position, and page ids outside [0, num_pages), are reported in the device error
 * word (rpa_device_error) and nothing is written for the affected rows.
 */
RPA_API rpa_status rpa_rotary_write_kv(rpa_plan_t plan, const void* q, const void* k,
                               const void* v, const rpa_rotary* rotary, void* q_out,
                               void* k_pool, void* v_pool, const int32_t* block_table,
                               const int32_t* cu_seqlens_q, const int32_t* seq_lens_k,
                               void* stream);

/*
 * rpa_forward -- the fused step: write the new tokens' K/V (when k_new/v_new are given)
 * and compute, for every query token t and query head hq,
 *     out[t, hq] = sum_j softmax_j(scale * q[t,hq] . K_j) V_j
 * over the keys j the token may see (causal mask; with group tables only keys whose
 * block -- of P tokens -- is listed for the row's KV group).  Exact attention: a
 * split-KV decode kernel with an LSE merge for short query rows, a tensor-core
 * (tcgen05/TMEM) kernel fed by TMA through the block table for the rest.
 *
 *   q                 device bf16 [T, Hq, D].
 *   k_new, v_new      device bf16 [T, Hkv, D], or both NULL when the cache already holds
 *                     the new tokens (e.g. after rpa_write_kv).  Given, a batch of short rows
 *                     and a mixed batch have the attention kernels write them into the pools
 *                     themselves (the cache write fused with attention, "Ragged Paged
 *                     Attention ..." Key ideas); a batch of only long rows, e4m3 pools and
 *                     device plans run a scatter kernel first.  Either way the pools hold
 *                     every new row when the call's work completes.
 *   k_pool, v_pool    device bf16 pools (written in place, then read: the alias rule
 *                     of the WebGPU page -- input and output cache are one buffer).
 *   block_table, cu_seqlens_q, seq_lens_k   as for rpa_write_kv.
 *   group_table       device int32 [B, Hkv, max_blocks_per_seq] of ascending logical
 *                     block indices (rpa_build_group_tables output), or NULL; requires
 *                     RPA_LAYOUT_HEAD_MAJOR and a plan made with opts.sparse = 1; or, with
 *                     opts.sparse = 2, rpa_build_qtile_tables' per-(query tile, query head)
 *                     tables.
 *   group_count       device int32 [B, Hkv] valid entries per table row, or NULL.
 *   scale             softmax scale (typically 1/sqrt(D)); any finite value.
 *   out               device bf16 [T, Hq, D] (round-to-nearest-even).
 *   lse               device fp32 [T, Hq] natural-log log-sum-exp of the scaled scores,
 *                     or NULL.  A row with no visible key gets out = 0, lse = -inf.
 *   workspace         device buffer of at least rpa_plan's workspace_bytes.
 * T == 0 returns RPA_OK and launches nothing.  Sequences with q_len == 0 are skipped.
 */
RPA_API rpa_status rpa_forward(rpa_plan_t plan, const void* q, const void* k_new, const void* v_new,
                       void* k_pool, void* v_pool, const int32_t* block_table,
                       const int32_t* cu_seqlens_q, const int32_t* seq_lens_k,
                       const int32_t* group_table, const int32_t* group_count, float scale,
                       void* out, float* lse, void* workspace, size_t workspace_bytes,
                       void* stream);

/*
 * rpa_forward_kv8 -- rpa_forward over an fp8 (e4m3) KV cache with per-KV-head scales.  Not
 * in the pages' shipped kernels: the WebGPU page's commit "FlashAttention: optional
 * seqlens_q input" lists the quantised KV cache under "Not in scope (deferred)"; this is
 * that extension: one byte per element halves the traffic of the bandwidth-bound decode path
 * and of the tensor-core kernel's K/V tiles.
 *
 *   k_pool, v_pool    device uint8 pools of e4m3 codes (1 sign, 4 exponent bits with bias
 *                     7, 3 mantissa bits; no infinities; 0x7F / 0xFF are NaN; largest
 *                     finite 448), in shape.layout with one byte per element.
 *   k_scale, v_scale  device fp32 [Hkv]: key j of KV head h is e4m3(k_pool[j, h]) * k_scale[h]
 *                     (the same for V).  Positive and finite.
 *   k_new, v_new      device bf16 [T, Hkv, D], or both NULL.  Each new element x is stored as
 *                     the e4m3 code nearest to fp32(x) / scale (IEEE fp32 division; ties to
 *                     the even code; magnitudes past 448 saturate to +-448).
 *   group_table, group_count  as for rpa_forward (plans made with opts.sparse = 1 or 2),
 *                     else NULL.
 *   the rest          as for rpa_forward.
 * Supported: head_dim 128.  Both attention kernels read the e4m3 pools in place and compute
 * on f16 operands (e4m3 -> f16 is exact; q is converted to f16, exact within f16's range,
 * so |q| must stay below 65504), with fp32 accumulation and P rounded to f16; k_scale[h] is
 * folded into the score scale and v_scale[h] into the output.  Host plans with rows for the
 * tensor-core kernel and device plans (rpa_plan_device) must be made with opts.kv_e4m3 = 1;
 * a device plan over e4m3 pools runs every batch class, so a step can be captured in a CUDA
 * graph.  Anything else returns RPA_ERR_UNSUPPORTED.
 */
RPA_API rpa_status rpa_forward_kv8(rpa_plan_t plan, const void* q, const void* k_new,
                                   const void* v_new, void* k_pool, void* v_pool,
                                   const float* k_scale, const float* v_scale,
                                   const int32_t* block_table, const int32_t* cu_seqlens_q,
                                   const int32_t* seq_lens_k, const int32_t* group_table,
                                   const int32_t* group_count, float scale, void* out,
                                   float* lse, void* workspace, size_t workspace_bytes,
                                   void* stream);

/*
 * rpa_forward_no_alloc -- rpa_forward for callers that cannot allocate device memory.
 * No counterpart in the pages: this is a convenience of this library.
 *
 * Who needs it: a host framework that owns all device memory -- a serving engine whose
 * allocator reserved the pool at start-up, or a plugin interface that passes the operator
 * only its inputs and outputs -- cannot hand rpa_forward a workspace, and a cudaMalloc on the
 * step's path would stall the stream or fail.  This entry point allocates nothing: the
 * step's scratch (the work lists copied from the plan and the split-KV decode partials) lives
 * in a fixed array of RPA_NO_ALLOC_WORKSPACE_BYTES that the library holds on every device
 * that loads it, until the process exits.
 *
 * Arguments, results and errors are those of rpa_forward minus the workspace.  A plan whose
 * rpa_plan workspace size exceeds RPA_NO_ALLOC_WORKSPACE_BYTES is rejected with
 * RPA_ERR_WORKSPACE_TOO_SMALL (use rpa_forward with a workspace for such batches).
 * The first call on a device looks up the array's device address (once per device, with
 * that device current); make that first call before any stream capture.
 * All calls share the one array: calls whose work overlaps on the GPU (different streams,
 * or different host threads on one device) race and must be serialised by the caller.  The
 * array keeps the last call's contents; nothing in it needs to start at zero, because every
 * call rewrites its work lists and every partial result before reading them.
 * The looked-up address is kept for the life of the process: after cudaDeviceReset (or any
 * other teardown of the device's primary context) it is stale, so do not call this entry
 * point on a device after resetting it.
 */
#define RPA_NO_ALLOC_WORKSPACE_BYTES ((size_t)8 << 20)

RPA_API rpa_status rpa_forward_no_alloc(rpa_plan_t plan, const void* q, const void* k_new,
                                        const void* v_new, void* k_pool, void* v_pool,
                                        const int32_t* block_table, const int32_t* cu_seqlens_q,
                                        const int32_t* seq_lens_k, const int32_t* group_table,
                                        const int32_t* group_count, float scale, void* out,
                                        float* lse, void* stream);

/* The size of rpa_forward_no_alloc's built-in scratch, RPA_NO_ALLOC_WORKSPACE_BYTES, as
 * compiled into the library (for bindings that do not read this header).  No CUDA call. */
RPA_API size_t rpa_no_alloc_workspace_bytes(void);

/*
 * rpa_build_group_tables -- block-union KV selection (CompactAttention, Core claim and
 * Fig. 3): for every sequence b and KV group g, the ascending list of KV blocks kb such
 * that some query head hq of the group (hq / (Hq/Hkv) == g) selects kb in some query
 * block: table[b, g, 0 .. count[b,g]-1]; remaining entries are set to -1.
 *
 *   mask    device uint8 [B, Hq, nqb, nkb], nonzero = selected.
 *   table   device int32 [B, Hkv, nkb].
 *   count   device int32 [B, Hkv].
 * Bit-exact and deterministic.  nkb <= 65536.
 */
RPA_API rpa_status rpa_build_group_tables(const uint8_t* mask, int32_t num_seqs, int32_t num_q_heads,
                                  int32_t num_kv_heads, int32_t num_q_blocks,
                                  int32_t num_kv_blocks, int32_t* table, int32_t* count,
                                  void* stream);

/*
 * rpa_build_qtile_tables -- per-(query tile, query head) KV block tables: row (b, hq, tile)
 * lists, ascending, the KV blocks kb that head hq selects in any query block of the
 * 128-query tile (query blocks tile * 128/q_block_rows ...); count[b, hq, tile] entries are
 * valid, the rest are -1.  This is the execution of a block-sparse kernel that works per
 * query block and head, for CompactAttention's execution-only ablation (Fig. 7c: the same
 * unioned mask, run block-sparse per query block vs. through per-group tables).  Pass the
 * tables to rpa_forward (as group_table / group_count) with a plan made with opts.sparse = 2:
 * the tensor-core kernel then runs one query head per CTA, each reading its own table.
 *
 *   mask          device uint8 [B, Hq, nqb, nkb], nonzero = selected.
 *   q_block_rows  query rows per mask block; must divide 128.
 *   table         device int32 [B, Hq, ntiles, nkb], ntiles = ceil(nqb * q_block_rows / 128),
 *                 which must equal ceil(max q_len / 128) of the plan; nkb = max_blocks_per_seq.
 *   count         device int32 [B, Hq, ntiles].
 */
RPA_API rpa_status rpa_build_qtile_tables(const uint8_t* mask, int32_t num_seqs,
                                          int32_t num_q_heads, int32_t num_q_blocks,
                                          int32_t num_kv_blocks, int32_t q_block_rows,
                                          int32_t* table, int32_t* count, void* stream);

/*
 * rpa_device_error -- read (and optionally clear) the library's device error word on the
 * current device.  Kernels never spin without bound: a wait that runs out records a code
 * here and the kernel returns early.  Synchronizes the device.  *code = 0 means no error;
 * otherwise an OR of: 1 decode wait ran out, 2 prefill wait ran out, 4 a page id outside
 * [0, num_pages) or a block index outside the table, 8 a position at or past the rotary
 * caches' max_position, 16 a device-planned step beyond its plan's limits.
 */
RPA_API rpa_status rpa_device_error(int32_t* code, int32_t clear);

/* rpa_status_string -- static description of a status code. */
RPA_API const char* rpa_status_string(rpa_status status);

/* rpa_last_error -- thread-local detail of the last failure on this thread ("" if none). */
RPA_API const char* rpa_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* RPA_H */
