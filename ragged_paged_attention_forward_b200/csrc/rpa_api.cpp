// C ABI of librpa.so (include/rpa.h): argument validation, the host planner and the launch
// sequence of one step.
//
// The planner is the distribution-aware part of "Ragged Paged Attention: A High-Performance
// and Flexible LLM Inference Kernel for TPU" (Key ideas): it classifies the batch (decode /
// prefill / mixed, with the q_len < 32 decode threshold of "[WebGPU] Optimized PagedAttention
// implementation (2/n)", "Correctness invariants") and slices the ragged batch into work
// items without padding: (sequence, key split) items for the split-KV decode kernel and
// (sequence, 128-query tile) items for the tensor-core kernel, heaviest first.  The work lists
// are built once on the host and copied into the caller's workspace by rpa_forward.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <cmath>
#include <new>
#include <string>
#include <vector>

#include "rpa.h"
#include "rpa_internal.h"

namespace rpa {

namespace {
thread_local std::string g_last_error;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int ilog2(int x) {
  int r = 0;
  while ((1 << r) < x) ++r;
  return r;
}
}  // namespace

void set_last_error(const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
}

}  // namespace rpa

using namespace rpa;

struct rpa_plan_s {
  rpa_shape shape;
  rpa_plan_options opts;
  int batch_class = RPA_CLASS_AUTO;
  int split_keys = 0;
  int decode_nt = 1;
  std::vector<DecodeItem> dec_items;
  std::vector<MergeRow> merge_rows;
  std::vector<PrefillTile> pf_tiles;
  int num_part_slots = 0;
  // workspace layout: [decode items][merge rows][prefill tiles] | [partial O][partial LSE]
  size_t off_dec = 0, off_merge = 0, off_pf = 0, meta_bytes = 0;
  size_t off_part_o = 0, off_part_lse = 0, ws_bytes = 0;
  std::vector<uint8_t> meta;  // host image of the metadata region
  // every list short enough to travel as kernel parameters: no work-list copy at all
  bool inline_lists = false;
  DecodeItemsInline dec_inline;
  MergeRowsInline merge_inline;
  PrefillTilesInline pf_inline;
  // pure decode plans fold the KV write into the decode kernel
  bool fuse_write = false;
  // host plans over bf16 pools with rows for both kernels (mixed batches): each attention
  // kernel writes its own rows' new K/V; only new rows that share a TMA box with older keys
  // (pf_straddle) need the scatter kernel first
  bool pf_straddle = false;
  int decode_skip_rows = 0;  // the scatter kernel skips sequences with q_len * G <= this
  // mixed batches: SMs of the persistent tensor-core grid beside the decode kernel (0: one
  // CTA per unit instead); see mixed_grid()
  int mixed_grid = 0;
  // device-planned plans: the lists are built on the device at every call, up to these caps
  bool device_mode = false;
  int max_kv_len = 0;
  int cap_items = 0, cap_rows = 0, cap_tiles = 0;
  // opts.sparse == 2: query tiles per sequence in the per-(query tile, head) tables
  int qtiles_per_seq = 0;
  size_t off_counts = 0;
  int launches_forward = 0;
  int launches_write = 0;
  // fork/join events of a mixed batch (created on first use, on the device of that call)
  cudaEvent_t fork_ev = nullptr;
  cudaEvent_t join_ev = nullptr;
  cudaEvent_t launched_ev = nullptr;  // the tensor-core grid of a split mixed step is resident
  ~rpa_plan_s() {
    if (fork_ev) cudaEventDestroy(fork_ev);
    if (join_ev) cudaEventDestroy(join_ev);
    if (launched_ev) cudaEventDestroy(launched_ev);
  }
};

#define RPA_FAIL(code, ...)            \
  do {                                 \
    rpa::set_last_error(__VA_ARGS__);  \
    return (code);                     \
  } while (0)

namespace {

rpa_status check_cuda(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return RPA_OK;
  rpa::set_last_error("%s: %s", what, cudaGetErrorString(e));
  return RPA_ERR_CUDA;
}

rpa_status validate_shape(const rpa_shape& s) {
  if (s.num_seqs < 0 || s.num_tokens < 0)
    RPA_FAIL(RPA_ERR_SHAPE, "num_seqs (%d) and num_tokens (%d) must be >= 0", s.num_seqs,
             s.num_tokens);
  if (s.num_q_heads <= 0 || s.num_kv_heads <= 0)
    RPA_FAIL(RPA_ERR_SHAPE, "head counts must be positive (Hq=%d, Hkv=%d)", s.num_q_heads,
             s.num_kv_heads);
  if (s.num_q_heads % s.num_kv_heads != 0)
    RPA_FAIL(RPA_ERR_SHAPE, "num_q_heads (%d) must be a multiple of num_kv_heads (%d)",
             s.num_q_heads, s.num_kv_heads);
  if (s.head_dim != 64 && s.head_dim != 128)
    RPA_FAIL(RPA_ERR_UNSUPPORTED, "head_dim %d is not supported (64 or 128)", s.head_dim);
  if (s.page_size < 16 || s.page_size > 256 || (s.page_size & (s.page_size - 1)) != 0)
    RPA_FAIL(RPA_ERR_UNSUPPORTED, "page_size %d must be a power of two in [16, 256]",
             s.page_size);
  if (s.num_pages <= 0) RPA_FAIL(RPA_ERR_SHAPE, "num_pages (%d) must be > 0", s.num_pages);
  if (s.max_blocks_per_seq <= 0)
    RPA_FAIL(RPA_ERR_SHAPE, "max_blocks_per_seq (%d) must be > 0", s.max_blocks_per_seq);
  if (s.layout != RPA_LAYOUT_SEQ_MAJOR && s.layout != RPA_LAYOUT_HEAD_MAJOR)
    RPA_FAIL(RPA_ERR_INVALID_ARG, "unknown layout %d", s.layout);
  if (s.causal != 0 && s.causal != 1) RPA_FAIL(RPA_ERR_INVALID_ARG, "causal must be 0 or 1");
  return RPA_OK;
}

// Decode items hold every query row of their sequence in the N dimension of the warp MMAs:
// q_len * G <= 32.
constexpr int kMaxDecodeRows = 32;

int auto_split_keys(long total_key_heads, int sms) {
  // aim for >= ~8 CTAs per SM (two resident, four waves) without splits under 256 keys
  const long target_ctas = (long)sms * 8;
  long s = total_key_heads / std::max(1L, target_ctas);
  s = (s + kDecodeStageKeys - 1) / kDecodeStageKeys * kDecodeStageKeys;
  s = std::max<long>(s, kMinSplitKeys);
  s = std::min<long>(s, kMaxSplitKeys);
  return (int)s;
}

// Mixed batches: the SMs that the tensor-core grid gets when it runs persistently beside the
// decode kernel, or 0 to launch it with one CTA per unit instead.  Both kernels want whole
// SMs (a tensor-core CTA holds one), so they share the GPU in space: the decode kernel is
// launched once every tensor-core CTA is resident and takes the other SMs, and each SM a
// persistent CTA leaves when its units are done.  Work model, in SM-microseconds (B200,
// measured): a 128-key tile of a unit costs kTileUs, a unit kUnitUs more; the decode kernel
// moves decode_gbps_per_sm per SM (42 GB/s of bf16 K/V, 33 GB/s of e4m3 codes: the whole-GPU
// rates over 148 SMs).  The balanced step time is both works over all SMs; the grid
// is the smallest whose static walk over the units (rounds of the grid size, alternating
// direction, as the kernel walks them) ends within 70% of it, so that its SMs pass to the
// decode kernel before the decode work runs out (on the mixed workload the step measured
// 0.463 / 0.455 / 0.444 / 0.465 ms with 64 / 72 / 80 / 88 SMs, 0.53 ms with a CTA per unit).  Batches where either part is small, or
// that are short, keep the unit-per-CTA launch.
int mixed_grid(const std::vector<PrefillTile>& tiles, const rpa_shape& s, int hpc,
               double decode_bytes, double decode_gbps_per_sm, int sms) {
  if (tiles.empty() || decode_bytes <= 0 || sms < 64) return 0;
  const double kTileUs = (s.head_dim == 128 ? 2.2 : 1.6) * (hpc == 2 ? 1.0 : 0.6);
  const double kUnitUs = 2.0;
  const int groups = s.num_q_heads / hpc;
  std::vector<double> cost;
  cost.reserve(tiles.size() * groups);
  double wp = 0;
  for (const PrefillTile& t : tiles) {
    const long past = t.kv_len - t.q_len;
    const long q_end = std::min(t.q_len, t.q_start + kPrefillTileRows);
    const long kv_hi = s.causal ? std::min<long>(t.kv_len, past + q_end) : t.kv_len;
    const double c = (double)((kv_hi + kPrefillTileKeys - 1) / kPrefillTileKeys) * kTileUs + kUnitUs;
    for (int g = 0; g < groups; ++g) cost.push_back(c);
    wp += c * groups;
  }
  const double wd = decode_bytes / (decode_gbps_per_sm * 1e3);  // bytes per us per SM
  const double total = (wp + wd) / sms;                         // balanced step, us
  if (total < 100.0 || wp < 0.15 * (wp + wd) || wd < 0.15 * (wp + wd) || cost.size() > 8192)
    return 0;
  const double target = 0.7 * total;
  auto makespan = [&](int n) {
    std::vector<double> fin(n, 0.0);
    for (size_t u = 0; u < cost.size(); ++u) {
      const int k = (int)(u / n), i = (int)(u % n);
      fin[(k & 1) ? n - 1 - i : i] += cost[u];
    }
    return *std::max_element(fin.begin(), fin.end());
  };
  int lo = 1, hi = sms - 32;  // the decode kernel keeps at least 32 SMs
  if (hi < lo || makespan(hi) > target) return 0;
  while (lo < hi) {  // the makespan falls as the grid grows (close enough to search)
    const int mid = (lo + hi) / 2;
    if (makespan(mid) <= target) hi = mid; else lo = mid + 1;
  }
  return lo;
}

}  // namespace

extern "C" {

const char* rpa_status_string(rpa_status s) {
  switch (s) {
    case RPA_OK: return "RPA_OK";
    case RPA_ERR_INVALID_ARG: return "RPA_ERR_INVALID_ARG";
    case RPA_ERR_UNSUPPORTED: return "RPA_ERR_UNSUPPORTED";
    case RPA_ERR_SHAPE: return "RPA_ERR_SHAPE";
    case RPA_ERR_WORKSPACE_TOO_SMALL: return "RPA_ERR_WORKSPACE_TOO_SMALL";
    case RPA_ERR_CUDA: return "RPA_ERR_CUDA";
    case RPA_ERR_DEVICE_CHECK: return "RPA_ERR_DEVICE_CHECK";
  }
  return "RPA_ERR_UNKNOWN";
}

const char* rpa_last_error(void) { return g_last_error.c_str(); }

rpa_status rpa_plan(const rpa_shape* shape, const int32_t* cu_seqlens_q,
                    const int32_t* seq_lens_k, const rpa_plan_options* opts,
                    rpa_plan_t* out_plan, size_t* workspace_bytes) {
  g_last_error.clear();
  if (!shape || !out_plan) RPA_FAIL(RPA_ERR_INVALID_ARG, "shape and out_plan must not be NULL");
  *out_plan = nullptr;
  rpa_status st = validate_shape(*shape);
  if (st != RPA_OK) return st;
  const rpa_shape& s = *shape;
  const int B = s.num_seqs;
  if (B > 0 && (!cu_seqlens_q || !seq_lens_k))
    RPA_FAIL(RPA_ERR_INVALID_ARG, "cu_seqlens_q and seq_lens_k (host arrays) are required");
  rpa_plan_options o;
  memset(&o, 0, sizeof(o));
  if (opts) o = *opts;
  for (int i = 0; i < 3; ++i)
    if (o.reserved[i] != 0) RPA_FAIL(RPA_ERR_INVALID_ARG, "plan option reserved[%d] != 0", i);
  if (o.wait_test_us < 0 || o.wait_test_us > 1000000)
    RPA_FAIL(RPA_ERR_INVALID_ARG, "opts.wait_test_us %d must be in [0, 1000000]", o.wait_test_us);
  if (o.kv_e4m3 < 0 || o.kv_e4m3 > 1)
    RPA_FAIL(RPA_ERR_INVALID_ARG, "opts.kv_e4m3 %d must be 0 or 1", o.kv_e4m3);
  if (o.kv_e4m3 && s.head_dim != 128)
    RPA_FAIL(RPA_ERR_UNSUPPORTED, "e4m3 pools need head_dim 128 (got %d)", s.head_dim);
  if (o.force_class < RPA_CLASS_AUTO || o.force_class > RPA_CLASS_MIXED)
    RPA_FAIL(RPA_ERR_INVALID_ARG, "unknown force_class %d", o.force_class);
  if (o.decode_split_keys != 0 &&
      (o.decode_split_keys % kDecodeStageKeys != 0 || o.decode_split_keys < kDecodeStageKeys ||
       o.decode_split_keys > kMaxSplitKeys))
    RPA_FAIL(RPA_ERR_INVALID_ARG, "decode_split_keys %d must be a multiple of %d in [%d, %d]",
             o.decode_split_keys, kDecodeStageKeys, kDecodeStageKeys, kMaxSplitKeys);
  if (o.sparse < 0 || o.sparse > 2)
    RPA_FAIL(RPA_ERR_INVALID_ARG, "opts.sparse %d must be 0, 1 or 2", o.sparse);
  if (o.sparse && s.layout != RPA_LAYOUT_HEAD_MAJOR)
    RPA_FAIL(RPA_ERR_UNSUPPORTED, "block-union tables need the KV-head-major layout");
  if (o.sparse && s.page_size > kMaxSparsePage)
    RPA_FAIL(RPA_ERR_UNSUPPORTED, "block-union tables need page_size <= %d", kMaxSparsePage);

  // ---- lengths
  if (B > 0) {
    if (cu_seqlens_q[0] != 0) RPA_FAIL(RPA_ERR_SHAPE, "cu_seqlens_q[0] must be 0");
    for (int b = 0; b < B; ++b) {
      const int q_len = cu_seqlens_q[b + 1] - cu_seqlens_q[b];
      if (q_len < 0) RPA_FAIL(RPA_ERR_SHAPE, "cu_seqlens_q is decreasing at %d", b);
      const int kv = seq_lens_k[b];
      if (kv < 0) RPA_FAIL(RPA_ERR_SHAPE, "seq_lens_k[%d] = %d < 0", b, kv);
      if (q_len > kv)
        RPA_FAIL(RPA_ERR_SHAPE, "sequence %d: q_len %d exceeds kv_len %d", b, q_len, kv);
      const long blocks = ((long)kv + s.page_size - 1) / s.page_size;
      if (blocks > s.max_blocks_per_seq)
        RPA_FAIL(RPA_ERR_SHAPE, "sequence %d: kv_len %d needs %ld pages > max_blocks_per_seq %d",
                 b, kv, blocks, s.max_blocks_per_seq);
    }
  }
  const int T = B > 0 ? cu_seqlens_q[B] : 0;
  if (T != s.num_tokens)
    RPA_FAIL(RPA_ERR_SHAPE, "cu_seqlens_q[B] = %d but num_tokens = %d", T, s.num_tokens);

  rpa_plan_s* plan = new (std::nothrow) rpa_plan_s();
  if (!plan) RPA_FAIL(RPA_ERR_INVALID_ARG, "out of host memory");
  plan->shape = s;
  plan->opts = o;

  // ---- classification (affects speed only, never results)
  const int G = s.num_q_heads / s.num_kv_heads;
  bool all_decode = true, all_prefill = true;
  for (int b = 0; b < B; ++b) {
    const int q_len = cu_seqlens_q[b + 1] - cu_seqlens_q[b];
    if (q_len == 0) continue;
    if (q_len > 1) all_decode = false;
    if (q_len < 32) all_prefill = false;
  }
  int cls = all_decode ? RPA_CLASS_DECODE : (all_prefill ? RPA_CLASS_PREFILL : RPA_CLASS_MIXED);
  if (o.force_class != RPA_CLASS_AUTO) cls = o.force_class;
  plan->batch_class = cls;

  // row routing: the split-KV decode kernel takes short rows whose query heads x tokens fit
  // the warp MMA's N (<= 16 for mixed batches, <= 32 when forced / pure decode)
  const int decode_rows_cap = (cls == RPA_CLASS_MIXED) ? 16 : kMaxDecodeRows;
  std::vector<int> to_decode(B, 0);
  long total_key_heads = 0;
  int max_rows = 0;
  for (int b = 0; b < B; ++b) {
    const int q_len = cu_seqlens_q[b + 1] - cu_seqlens_q[b];
    if (q_len == 0) continue;
    const bool dec = !o.sparse && cls != RPA_CLASS_PREFILL && q_len * G <= decode_rows_cap;
    to_decode[b] = dec ? 1 : 0;
    if (dec) {
      total_key_heads += (long)seq_lens_k[b] * s.num_kv_heads;
      max_rows = std::max(max_rows, q_len * G);
    }
  }
  plan->decode_nt = max_rows <= 8 ? 1 : (max_rows <= 16 ? 2 : 4);
  plan->split_keys = o.decode_split_keys ? o.decode_split_keys
                                         : auto_split_keys(total_key_heads, device_sm_count());

  // ---- decode items and merge rows
  int slots = 0;
  for (int b = 0; b < B; ++b) {
    if (!to_decode[b]) continue;
    const int t0 = cu_seqlens_q[b];
    const int q_len = cu_seqlens_q[b + 1] - t0;
    const int kv = seq_lens_k[b];
    const int nsplit = (kv + plan->split_keys - 1) / plan->split_keys;
    for (int sp = 0; sp < nsplit; ++sp) {
      DecodeItem it;
      it.seq = b;
      it.t0 = t0;
      it.q_len = q_len;
      it.kv_len = kv;
      it.k_begin = sp * plan->split_keys;
      it.k_end = std::min(kv, (sp + 1) * plan->split_keys);
      it.part_slot = nsplit > 1 ? slots + sp : -1;
      it.pad = 0;
      plan->dec_items.push_back(it);
    }
    if (nsplit > 1) {
      for (int i = 0; i < q_len; ++i) plan->merge_rows.push_back(MergeRow{t0 + i, i, slots, nsplit});
      slots += nsplit;
    }
  }
  plan->num_part_slots = slots;
  // longest items first so the tail of the grid is short
  std::stable_sort(plan->dec_items.begin(), plan->dec_items.end(),
                   [](const DecodeItem& a, const DecodeItem& b) {
                     return (a.k_end - a.k_begin) > (b.k_end - b.k_begin);
                   });

  // ---- prefill tiles (heaviest first: most visible keys)
  for (int b = 0; b < B; ++b)
    plan->qtiles_per_seq = std::max(plan->qtiles_per_seq,
                                    (cu_seqlens_q[b + 1] - cu_seqlens_q[b] + kPrefillTileRows - 1) /
                                        kPrefillTileRows);
  for (int b = 0; b < B; ++b) {
    const int t0 = cu_seqlens_q[b];
    const int q_len = cu_seqlens_q[b + 1] - t0;
    if (q_len == 0 || to_decode[b]) continue;
    for (int qs = 0; qs < q_len; qs += kPrefillTileRows) {
      PrefillTile t;
      t.seq = b;
      t.t0 = t0;
      t.q_len = q_len;
      t.kv_len = seq_lens_k[b];
      t.q_start = qs;
      t.pad[0] = t.pad[1] = t.pad[2] = 0;
      plan->pf_tiles.push_back(t);
    }
  }
  auto work = [&](const PrefillTile& t) {
    const long past = t.kv_len - t.q_len;
    const long q_end = std::min(t.q_len, t.q_start + kPrefillTileRows);
    return s.causal ? std::min<long>(t.kv_len, past + q_end) : (long)t.kv_len;
  };
  std::stable_sort(plan->pf_tiles.begin(), plan->pf_tiles.end(),
                   [&](const PrefillTile& a, const PrefillTile& b) { return work(a) > work(b); });

  // ---- workspace layout
  size_t off = 0;
  plan->off_dec = off;
  off = align_up(off + plan->dec_items.size() * sizeof(DecodeItem), 256);
  plan->off_merge = off;
  off = align_up(off + plan->merge_rows.size() * sizeof(MergeRow), 256);
  plan->off_pf = off;
  off = align_up(off + plan->pf_tiles.size() * sizeof(PrefillTile), 256);
  plan->meta_bytes = off;
  const size_t rows_per_item = 8 * plan->decode_nt;
  plan->off_part_o = off;
  off = align_up(off + (size_t)slots * s.num_kv_heads * rows_per_item * s.head_dim * 4, 256);
  plan->off_part_lse = off;
  off = align_up(off + (size_t)slots * s.num_kv_heads * rows_per_item * 4, 256);
  plan->ws_bytes = std::max<size_t>(off, 256);
  plan->meta.assign(plan->meta_bytes, 0);
  if (!plan->dec_items.empty())
    memcpy(plan->meta.data() + plan->off_dec, plan->dec_items.data(),
           plan->dec_items.size() * sizeof(DecodeItem));
  if (!plan->merge_rows.empty())
    memcpy(plan->meta.data() + plan->off_merge, plan->merge_rows.data(),
           plan->merge_rows.size() * sizeof(MergeRow));
  if (!plan->pf_tiles.empty())
    memcpy(plan->meta.data() + plan->off_pf, plan->pf_tiles.data(),
           plan->pf_tiles.size() * sizeof(PrefillTile));

  plan->inline_lists = plan->dec_items.size() <= (size_t)kInlineItems &&
                       plan->merge_rows.size() <= (size_t)kInlineItems &&
                       plan->pf_tiles.size() <= (size_t)kInlineItems;
  memset(&plan->dec_inline, 0, sizeof(plan->dec_inline));
  memset(&plan->merge_inline, 0, sizeof(plan->merge_inline));
  memset(&plan->pf_inline, 0, sizeof(plan->pf_inline));
  if (plan->inline_lists) {
    std::copy(plan->dec_items.begin(), plan->dec_items.end(), plan->dec_inline.v);
    std::copy(plan->merge_rows.begin(), plan->merge_rows.end(), plan->merge_inline.v);
    std::copy(plan->pf_tiles.begin(), plan->pf_tiles.end(), plan->pf_inline.v);
  }
  plan->fuse_write = plan->pf_tiles.empty() && !plan->dec_items.empty();
  {
    const int box = std::min(s.page_size, kPrefillTileKeys);
    for (int b = 0; b < B; ++b) {
      const int q_len = cu_seqlens_q[b + 1] - cu_seqlens_q[b];
      if (q_len > 0 && !to_decode[b] && (seq_lens_k[b] - q_len) % box != 0)
        plan->pf_straddle = true;
    }
    plan->decode_skip_rows = plan->dec_items.empty() ? 0 : decode_rows_cap;
  }
  if (!plan->pf_tiles.empty() && !plan->dec_items.empty() && !o.sparse) {
    const int elem = o.kv_e4m3 ? 1 : 2;  // bytes per K/V element the decode kernel reads
    double dbytes = 0;
    for (const DecodeItem& it : plan->dec_items)
      dbytes += (double)(it.k_end - it.k_begin) * s.num_kv_heads * s.head_dim * 2 * elem;
    const int G = s.num_q_heads / s.num_kv_heads;
    plan->mixed_grid = mixed_grid(plan->pf_tiles, s, (G & 1) == 0 ? 2 : 1, dbytes,
                                  o.kv_e4m3 ? 33.0 : 42.0, device_sm_count());
  }
  plan->launches_write = T > 0 ? 1 : 0;
  const bool pf_writes = !plan->pf_tiles.empty() && !plan->dec_items.empty() && !o.kv_e4m3;
  const int write_in_forward =
      plan->fuse_write ? 0 : (pf_writes ? (plan->pf_straddle ? 1 : 0) : plan->launches_write);
  plan->launches_forward = write_in_forward +
                           (plan->dec_items.empty() ? 0 : 1) +
                           (plan->merge_rows.empty() ? 0 : 1) +
                           (plan->pf_tiles.empty() ? 0 : 1);
  *out_plan = plan;
  if (workspace_bytes) *workspace_bytes = plan->ws_bytes;
  return RPA_OK;
}

rpa_status rpa_plan_device(const rpa_shape* shape, int32_t max_kv_len,
                           const rpa_plan_options* opts, rpa_plan_t* out_plan,
                           size_t* workspace_bytes) {
  g_last_error.clear();
  if (!shape || !out_plan) RPA_FAIL(RPA_ERR_INVALID_ARG, "shape and out_plan must not be NULL");
  *out_plan = nullptr;
  rpa_status st = validate_shape(*shape);
  if (st != RPA_OK) return st;
  const rpa_shape& s = *shape;
  rpa_plan_options o;
  memset(&o, 0, sizeof(o));
  if (opts) o = *opts;
  for (int i = 0; i < 3; ++i)
    if (o.reserved[i] != 0) RPA_FAIL(RPA_ERR_INVALID_ARG, "plan option reserved[%d] != 0", i);
  if (o.wait_test_us < 0 || o.wait_test_us > 1000000)
    RPA_FAIL(RPA_ERR_INVALID_ARG, "opts.wait_test_us %d must be in [0, 1000000]", o.wait_test_us);
  if (o.sparse) RPA_FAIL(RPA_ERR_UNSUPPORTED, "device-planned steps take no group tables");
  if (o.wait_test_us) RPA_FAIL(RPA_ERR_UNSUPPORTED, "opts.wait_test_us: host plans only");
  if (o.kv_e4m3 && s.head_dim != 128)
    RPA_FAIL(RPA_ERR_UNSUPPORTED, "e4m3 pools need head_dim 128 (got %d)", s.head_dim);
  if (o.force_class != RPA_CLASS_AUTO)
    RPA_FAIL(RPA_ERR_UNSUPPORTED, "device-planned steps choose their kernels per sequence");
  if (o.decode_split_keys != 0 &&
      (o.decode_split_keys % kDecodeStageKeys != 0 || o.decode_split_keys < kDecodeStageKeys ||
       o.decode_split_keys > kMaxSplitKeys))
    RPA_FAIL(RPA_ERR_INVALID_ARG, "decode_split_keys %d must be a multiple of %d in [%d, %d]",
             o.decode_split_keys, kDecodeStageKeys, kDecodeStageKeys, kMaxSplitKeys);
  if (max_kv_len < 1 || (long)max_kv_len > (long)s.max_blocks_per_seq * s.page_size)
    RPA_FAIL(RPA_ERR_SHAPE, "max_kv_len %d must be in [1, max_blocks_per_seq * page_size]",
             max_kv_len);
  rpa_plan_s* plan = new (std::nothrow) rpa_plan_s();
  if (!plan) RPA_FAIL(RPA_ERR_INVALID_ARG, "out of host memory");
  plan->shape = s;
  plan->opts = o;
  plan->device_mode = true;
  plan->max_kv_len = max_kv_len;
  plan->batch_class = RPA_CLASS_AUTO;
  // a sequence goes to the decode kernel when its query heads x tokens fit the smallest MMA
  // column count that holds one token's group (8, 16 or 32)
  const int G = s.num_q_heads / s.num_kv_heads;
  plan->decode_nt = G <= 8 ? 1 : (G <= 16 ? 2 : 4);
  const int B = s.num_seqs;
  // split size for an average context of max_kv_len / 2, as the host planner would pick it
  plan->split_keys = o.decode_split_keys
                         ? o.decode_split_keys
                         : auto_split_keys((long)B * (max_kv_len / 2) * s.num_kv_heads,
                                           device_sm_count());
  const long splits = (max_kv_len + plan->split_keys - 1) / plan->split_keys;
  plan->cap_items = (int)std::min<long>((long)B * splits, 1L << 24);
  plan->cap_rows = std::max(s.num_tokens, 1);
  // a sequence reaches the tensor-core kernel only with q_len * G > 8 * decode_nt, i.e. with
  // at least qmin tokens, so at most T / qmin sequences add a partial tile each: a bound far
  // below T / 128 + B for decode-heavy steps, which keeps the grid of early-exiting CTAs small
  const int qmin = 8 * plan->decode_nt / G + 1;
  plan->cap_tiles = (s.num_tokens + kPrefillTileRows - 1) / kPrefillTileRows +
                    std::min(B, s.num_tokens / qmin);
  size_t off = 0;
  plan->off_counts = off;
  off = align_up(off + 16, 256);
  plan->off_dec = off;
  off = align_up(off + (size_t)plan->cap_items * sizeof(DecodeItem), 256);
  plan->off_merge = off;
  off = align_up(off + (size_t)plan->cap_rows * sizeof(MergeRow), 256);
  plan->off_pf = off;
  off = align_up(off + (size_t)plan->cap_tiles * sizeof(PrefillTile), 256);
  const size_t rows_per_item = 8 * plan->decode_nt;
  plan->off_part_o = off;
  off = align_up(off + (size_t)plan->cap_items * s.num_kv_heads * rows_per_item * s.head_dim * 4,
                 256);
  plan->off_part_lse = off;
  off = align_up(off + (size_t)plan->cap_items * s.num_kv_heads * rows_per_item * 4, 256);
  plan->ws_bytes = off;
  plan->launches_write = 1;
  // planner, KV write, tensor-core, decode, merge
  plan->launches_forward = 5;
  *out_plan = plan;
  if (workspace_bytes) *workspace_bytes = plan->ws_bytes;
  return RPA_OK;
}

rpa_status rpa_plan_get_info(rpa_plan_t plan, rpa_plan_info* info) {
  if (!plan || !info) RPA_FAIL(RPA_ERR_INVALID_ARG, "plan and info must not be NULL");
  memset(info, 0, sizeof(*info));
  info->batch_class = plan->batch_class;
  info->num_decode_items = (int32_t)plan->dec_items.size();
  info->num_prefill_tiles = (int32_t)plan->pf_tiles.size();
  info->num_merge_rows = (int32_t)plan->merge_rows.size();
  info->launches_forward = plan->launches_forward;
  info->launches_write = plan->launches_write;
  info->decode_split_keys = plan->split_keys;
  info->tensor_core_grid = plan->mixed_grid;
  info->workspace_bytes = plan->ws_bytes;
  if (plan->device_mode) {  // the caps the device-built lists may reach
    info->num_decode_items = plan->cap_items;
    info->num_prefill_tiles = plan->cap_tiles;
    info->num_merge_rows = plan->cap_rows;
  }
  return RPA_OK;
}

void rpa_plan_destroy(rpa_plan_t plan) { delete plan; }

static rpa_status write_kv_impl(rpa_plan_t plan, const void* k_new, const void* v_new,
                                void* k_pool, void* v_pool, const int32_t* block_table,
                                const int32_t* cu_seqlens_q, const int32_t* seq_lens_k,
                                cudaStream_t stream, int skip_rows_upto = 0,
                                const float* k_scale = nullptr,
                                const float* v_scale = nullptr, int below_box = 0) {
  const rpa_shape& s = plan->shape;
  int* err = nullptr;
  rpa_status st = check_cuda(device_error_word(&err), "device error word");
  if (st != RPA_OK) return st;
  WriteLaunch w{};
  w.k_new = static_cast<const uint16_t*>(k_new);
  w.v_new = static_cast<const uint16_t*>(v_new);
  w.k_pool = k_pool;
  w.v_pool = v_pool;
  w.kv8 = k_scale != nullptr ? 1 : 0;
  w.k_scale = k_scale;
  w.v_scale = v_scale;
  w.block_table = block_table;
  w.cu_seqlens_q = cu_seqlens_q;
  w.seq_lens_k = seq_lens_k;
  w.num_seqs = s.num_seqs;
  w.num_tokens = s.num_tokens;
  w.num_kv_heads = s.num_kv_heads;
  w.head_dim = s.head_dim;
  w.page_size = s.page_size;
  w.max_blocks = s.max_blocks_per_seq;
  w.layout = s.layout;
  w.num_pages = s.num_pages;
  w.tokens_on_device = plan->device_mode ? 1 : 0;
  w.skip_rows_upto = skip_rows_upto;
  w.group = s.num_q_heads / s.num_kv_heads;
  w.below_box = below_box;
  w.err = err;
  return check_cuda(launch_write_kv(w, stream), "write_kv launch");
}

static rpa_status check_common(rpa_plan_t plan, const void* k_pool, const void* v_pool,
                               const int32_t* block_table, const int32_t* cu_seqlens_q,
                               const int32_t* seq_lens_k) {
  if (!plan) RPA_FAIL(RPA_ERR_INVALID_ARG, "plan must not be NULL");
  if (!k_pool || !v_pool || !block_table || !cu_seqlens_q || !seq_lens_k)
    RPA_FAIL(RPA_ERR_INVALID_ARG, "pools, block_table, cu_seqlens_q and seq_lens_k are required");
  if (!aligned16(k_pool) || !aligned16(v_pool))
    RPA_FAIL(RPA_ERR_INVALID_ARG, "k_pool / v_pool must be 16-byte aligned");
  return RPA_OK;
}

rpa_status rpa_write_kv(rpa_plan_t plan, const void* k_new, const void* v_new, void* k_pool,
                        void* v_pool, const int32_t* block_table, const int32_t* cu_seqlens_q,
                        const int32_t* seq_lens_k, void* workspace, size_t workspace_bytes,
                        void* stream) {
  (void)workspace;
  (void)workspace_bytes;
  g_last_error.clear();
  rpa_status st = check_common(plan, k_pool, v_pool, block_table, cu_seqlens_q, seq_lens_k);
  if (st != RPA_OK) return st;
  if (plan->shape.num_tokens == 0) return RPA_OK;
  if (!k_new || !v_new) RPA_FAIL(RPA_ERR_INVALID_ARG, "k_new and v_new are required");
  if (!aligned16(k_new) || !aligned16(v_new))
    RPA_FAIL(RPA_ERR_INVALID_ARG, "k_new / v_new must be 16-byte aligned");
  return write_kv_impl(plan, k_new, v_new, k_pool, v_pool, block_table, cu_seqlens_q,
                       seq_lens_k, static_cast<cudaStream_t>(stream));
}

rpa_status rpa_write_kv8(rpa_plan_t plan, const void* k_new, const void* v_new, void* k_pool,
                         void* v_pool, const float* k_scale, const float* v_scale,
                         const int32_t* block_table, const int32_t* cu_seqlens_q,
                         const int32_t* seq_lens_k, void* stream) {
  g_last_error.clear();
  rpa_status st = check_common(plan, k_pool, v_pool, block_table, cu_seqlens_q, seq_lens_k);
  if (st != RPA_OK) return st;
  if (plan->shape.head_dim % 16 != 0)
    RPA_FAIL(RPA_ERR_UNSUPPORTED, "e4m3 pools need head_dim a multiple of 16");
  if (plan->shape.num_tokens == 0) return RPA_OK;
  if (!k_new || !v_new) RPA_FAIL(RPA_ERR_INVALID_ARG, "k_new and v_new are required");
  if (!aligned16(k_new) || !aligned16(v_new))
    RPA_FAIL(RPA_ERR_INVALID_ARG, "k_new / v_new must be 16-byte aligned");
  if (!k_scale || !v_scale) RPA_FAIL(RPA_ERR_INVALID_ARG, "k_scale and v_scale are required");
  if ((reinterpret_cast<uintptr_t>(k_scale) & 3u) || (reinterpret_cast<uintptr_t>(v_scale) & 3u))
    RPA_FAIL(RPA_ERR_INVALID_ARG, "k_scale / v_scale must be 4-byte aligned");
  return write_kv_impl(plan, k_new, v_new, k_pool, v_pool, block_table, cu_seqlens_q,
                       seq_lens_k, static_cast<cudaStream_t>(stream), 0, k_scale, v_scale);
}

rpa_status rpa_rotary_write_kv(rpa_plan_t plan, const void* q, const void* k, const void* v,
                               const rpa_rotary* rotary, void* q_out, void* k_pool,
                               void* v_pool, const int32_t* block_table,
                               const int32_t* cu_seqlens_q, const int32_t* seq_lens_k,
                               void* stream) {
  g_last_error.clear();
  rpa_status st = check_common(plan, k_pool, v_pool, block_table, cu_seqlens_q, seq_lens_k);
  if (st != RPA_OK) return st;
  const rpa_shape& s = plan->shape;
  if (s.num_tokens == 0) return RPA_OK;
  if (!q || !q_out) RPA_FAIL(RPA_ERR_INVALID_ARG, "q and q_out are required");
  if ((k == nullptr) != (v == nullptr))
    RPA_FAIL(RPA_ERR_INVALID_ARG, "k and v must both be given or both be NULL (packed input)");
  if (!aligned16(q) || !aligned16(q_out) || (k && (!aligned16(k) || !aligned16(v))))
    RPA_FAIL(RPA_ERR_INVALID_ARG, "q, k, v and q_out must be 16-byte aligned");
  const size_t q_row = (size_t)(k ? s.num_q_heads : s.num_q_heads + 2 * s.num_kv_heads);
  const size_t q_bytes = (size_t)s.num_tokens * q_row * s.head_dim * 2;
  const size_t out_bytes = (size_t)s.num_tokens * s.num_q_heads * s.head_dim * 2;
  const uintptr_t qa = reinterpret_cast<uintptr_t>(q), oa = reinterpret_cast<uintptr_t>(q_out);
  if (qa < oa + out_bytes && oa < qa + q_bytes)
    RPA_FAIL(RPA_ERR_INVALID_ARG, "q_out must not overlap q");
  RotaryLaunch r{};
  r.cos = r.sin = nullptr;
  r.max_pos = 0;
  r.rotary_dim = 0;
  r.interleaved = 0;
  if (rotary) {
    const rpa_rotary& ro = *rotary;
    if (ro.reserved != 0) RPA_FAIL(RPA_ERR_INVALID_ARG, "rotary.reserved != 0");
    if (!ro.cos_cache || !ro.sin_cache)
      RPA_FAIL(RPA_ERR_INVALID_ARG, "rotation needs cos_cache and sin_cache");
    if (!aligned16(ro.cos_cache) || !aligned16(ro.sin_cache))
      RPA_FAIL(RPA_ERR_INVALID_ARG, "cos_cache / sin_cache must be 16-byte aligned");
    if (ro.rotary_dim < 16 || ro.rotary_dim % 16 != 0 || ro.rotary_dim > s.head_dim)
      RPA_FAIL(RPA_ERR_UNSUPPORTED, "rotary_dim %d must be a multiple of 16 in [16, %d]",
               ro.rotary_dim, s.head_dim);
    if (ro.max_position <= 0)
      RPA_FAIL(RPA_ERR_INVALID_ARG, "max_position %d must be positive", ro.max_position);
    if (ro.interleaved != 0 && ro.interleaved != 1)
      RPA_FAIL(RPA_ERR_INVALID_ARG, "interleaved must be 0 or 1");
    r.cos = static_cast<const uint16_t*>(ro.cos_cache);
    r.sin = static_cast<const uint16_t*>(ro.sin_cache);
    r.max_pos = ro.max_position;
    r.rotary_dim = ro.rotary_dim;
    r.interleaved = ro.interleaved;
  }
  int* err = nullptr;
  st = check_cuda(device_error_word(&err), "device error word");
  if (st != RPA_OK) return st;
  r.q = static_cast<const uint16_t*>(q);
  r.k = static_cast<const uint16_t*>(k);
  r.v = static_cast<const uint16_t*>(v);
  r.q_out = static_cast<uint16_t*>(q_out);
  r.k_pool = static_cast<uint16_t*>(k_pool);
  r.v_pool = static_cast<uint16_t*>(v_pool);
  r.block_table = block_table;
  r.cu_seqlens_q = cu_seqlens_q;
  r.seq_lens_k = seq_lens_k;
  r.num_seqs = s.num_seqs;
  r.num_tokens = s.num_tokens;
  r.num_q_heads = s.num_q_heads;
  r.num_kv_heads = s.num_kv_heads;
  r.head_dim = s.head_dim;
  r.page_size = s.page_size;
  r.max_blocks = s.max_blocks_per_seq;
  r.layout = s.layout;
  r.num_pages = s.num_pages;
  r.err = err;
  return check_cuda(launch_rotary_write(r, static_cast<cudaStream_t>(stream)),
                    "rotary write launch");
}

// The fused step for bf16 pools (rpa_forward) and for e4m3 pools (rpa_forward_kv8, kv8 =
// true, with per-KV-head scales; decode-class plans only, checked by the caller).
static rpa_status forward_impl(rpa_plan_t plan, const void* q, const void* k_new,
                               const void* v_new, void* k_pool, void* v_pool,
                               const int32_t* block_table, const int32_t* cu_seqlens_q,
                               const int32_t* seq_lens_k, const int32_t* group_table,
                               const int32_t* group_count, float scale, void* out, float* lse,
                               void* workspace, size_t workspace_bytes, void* stream_,
                               bool kv8, const float* k_scale, const float* v_scale) {
  rpa_status st = check_common(plan, k_pool, v_pool, block_table, cu_seqlens_q, seq_lens_k);
  if (st != RPA_OK) return st;
  const rpa_shape& s = plan->shape;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (s.num_tokens == 0) return RPA_OK;
  if (!q || !out) RPA_FAIL(RPA_ERR_INVALID_ARG, "q and out are required");
  if (!aligned16(q) || !aligned16(out))
    RPA_FAIL(RPA_ERR_INVALID_ARG, "q / out must be 16-byte aligned");
  if ((k_new == nullptr) != (v_new == nullptr))
    RPA_FAIL(RPA_ERR_INVALID_ARG, "k_new and v_new must both be given or both be NULL");
  if (k_new && (!aligned16(k_new) || !aligned16(v_new)))
    RPA_FAIL(RPA_ERR_INVALID_ARG, "k_new / v_new must be 16-byte aligned");
  if ((group_table == nullptr) != (group_count == nullptr))
    RPA_FAIL(RPA_ERR_INVALID_ARG, "group_table and group_count go together");
  if (group_table && s.layout != RPA_LAYOUT_HEAD_MAJOR)
    RPA_FAIL(RPA_ERR_INVALID_ARG, "group tables need the KV-head-major layout");
  if ((group_table != nullptr) != (plan->opts.sparse != 0))
    RPA_FAIL(RPA_ERR_INVALID_ARG,
             "tables must be given exactly when the plan was made with opts.sparse = 1 or 2");
  if (!std::isfinite(scale)) RPA_FAIL(RPA_ERR_INVALID_ARG, "scale must be finite");
  if (!workspace || workspace_bytes < plan->ws_bytes)
    RPA_FAIL(RPA_ERR_WORKSPACE_TOO_SMALL, "workspace of %zu bytes needed, %zu given",
             plan->ws_bytes, workspace ? workspace_bytes : (size_t)0);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    RPA_FAIL(RPA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");

  // A mixed batch over bf16 pools (host plan): each attention kernel writes its own rows' new
  // K/V (the cache write fused with attention); the scatter kernel runs first only for new
  // rows that share a TMA box with older keys.  A batch of only long rows keeps the scatter
  // kernel: measured, it is faster than the tensor-core kernel's own copy there.
  const bool fuse_pf = k_new && !kv8 && !plan->device_mode && !plan->pf_tiles.empty() &&
                       !plan->dec_items.empty();
  const int fuse_box = std::min(s.page_size, kPrefillTileKeys);
  if (k_new && !plan->device_mode) {
    if (fuse_pf) {
      if (plan->pf_straddle) {
        st = write_kv_impl(plan, k_new, v_new, k_pool, v_pool, block_table, cu_seqlens_q,
                           seq_lens_k, stream, plan->decode_skip_rows, nullptr, nullptr,
                           fuse_box);
        if (st != RPA_OK) return st;
      }
    } else if (!plan->fuse_write) {
      st = write_kv_impl(plan, k_new, v_new, k_pool, v_pool, block_table, cu_seqlens_q,
                         seq_lens_k, stream, 0, kv8 ? k_scale : nullptr,
                         kv8 ? v_scale : nullptr);
      if (st != RPA_OK) return st;
    }
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (plan->meta_bytes > 0 && !plan->inline_lists) {
    st = check_cuda(cudaMemcpyAsync(ws, plan->meta.data(), plan->meta_bytes,
                                    cudaMemcpyHostToDevice, stream),
                    "work-list copy");
    if (st != RPA_OK) return st;
  }
  int* err = nullptr;
  st = check_cuda(device_error_word(&err), "device error word");
  if (st != RPA_OK) return st;

  PagedKV kv;
  kv.k_pool = k_pool;
  kv.v_pool = v_pool;
  kv.block_table = block_table;
  kv.layout = s.layout;
  kv.page_size = s.page_size;
  kv.log2_page = ilog2(s.page_size);
  kv.max_blocks = s.max_blocks_per_seq;
  kv.num_kv_heads = s.num_kv_heads;
  kv.num_pages = s.num_pages;
  kv.kv8 = kv8 ? 1 : 0;
  const float scale_log2 = scale * 1.4426950408889634f;

  if (plan->device_mode) {
    // the lists are built from the device lengths first; every kernel then runs its
    // largest grid, and CTAs past the step's counts return at once
    int32_t* counts = reinterpret_cast<int32_t*>(ws + plan->off_counts);
    PlanDeviceLaunch pl{};
    pl.cu_seqlens_q = cu_seqlens_q;
    pl.seq_lens_k = seq_lens_k;
    pl.num_seqs = s.num_seqs;
    pl.max_tokens = s.num_tokens;
    pl.max_kv_len = plan->max_kv_len;
    pl.num_q_heads = s.num_q_heads;
    pl.num_kv_heads = s.num_kv_heads;
    pl.causal = s.causal;
    pl.split_keys = plan->split_keys;
    pl.decode_rows = 8 * plan->decode_nt;
    pl.cap_items = plan->cap_items;
    pl.cap_rows = plan->cap_rows;
    pl.cap_tiles = plan->cap_tiles;
    pl.items = reinterpret_cast<DecodeItem*>(ws + plan->off_dec);
    pl.rows = reinterpret_cast<MergeRow*>(ws + plan->off_merge);
    pl.tiles = reinterpret_cast<PrefillTile*>(ws + plan->off_pf);
    pl.counts = counts;
    pl.err = err;
    st = check_cuda(launch_plan_device(pl, stream), "device planner launch");
    if (st != RPA_OK) return st;
    // both kernel families: the tensor-core kernel on the side stream, forked after the
    // planner, the decode kernel and the merge on the caller's stream; joined at the end.
    cudaStream_t pf_stream = stream;
    st = check_cuda(side_stream(stream, &pf_stream), "side stream");
    if (st != RPA_OK) return st;
    if (!plan->fork_ev) {
      st = check_cuda(cudaEventCreateWithFlags(&plan->fork_ev, cudaEventDisableTiming),
                      "event create");
      if (st != RPA_OK) return st;
      st = check_cuda(cudaEventCreateWithFlags(&plan->join_ev, cudaEventDisableTiming),
                      "event create");
      if (st != RPA_OK) return st;
    }
    st = check_cuda(cudaEventRecord(plan->fork_ev, stream), "fork record");
    if (st != RPA_OK) return st;
    st = check_cuda(cudaStreamWaitEvent(pf_stream, plan->fork_ev, 0), "fork wait");
    if (st != RPA_OK) return st;
    // new tokens: the decode kernel writes those of its own rows (as for host plans); the
    // scatter kernel, on the side stream ahead of the tensor-core kernel, writes the rest
    if (k_new) {
      st = write_kv_impl(plan, k_new, v_new, k_pool, v_pool, block_table, cu_seqlens_q,
                         seq_lens_k, pf_stream, 8 * plan->decode_nt, kv8 ? k_scale : nullptr,
                         kv8 ? v_scale : nullptr);
      if (st != RPA_OK) return st;
    }
    PrefillLaunch p{};
    p.tiles = pl.tiles;
    p.num_tiles = plan->cap_tiles;
    p.count = counts + 2;
    p.q = static_cast<const uint16_t*>(q);
    p.num_tokens = s.num_tokens;
    p.num_q_heads = s.num_q_heads;
    p.num_kv_heads = s.num_kv_heads;
    p.head_dim = s.head_dim;
    p.causal = s.causal;
    p.scale_log2 = scale_log2;
    p.out = static_cast<uint16_t*>(out);
    p.lse = lse;
    p.err = err;
    p.kv = kv;
    p.k_scale = kv8 ? k_scale : nullptr;
    p.v_scale = kv8 ? v_scale : nullptr;
    st = check_cuda(launch_prefill(p, &plan->pf_inline, pf_stream), "prefill launch");
    if (st != RPA_OK) return st;
    DecodeLaunch d{};
    d.items = pl.items;
    d.num_items = plan->cap_items;
    d.count = counts;
    d.rows_per_item = 8 * plan->decode_nt;
    d.q = static_cast<const uint16_t*>(q);
    d.num_q_heads = s.num_q_heads;
    d.num_kv_heads = s.num_kv_heads;
    d.head_dim = s.head_dim;
    d.causal = s.causal;
    d.scale_log2 = scale_log2;
    d.out = static_cast<uint16_t*>(out);
    d.lse = lse;
    d.part_o = reinterpret_cast<float*>(ws + plan->off_part_o);
    d.part_lse = reinterpret_cast<float*>(ws + plan->off_part_lse);
    d.err = err;
    d.kv = kv;
    d.k_new = static_cast<const uint16_t*>(k_new);
    d.v_new = static_cast<const uint16_t*>(v_new);
    d.k_pool_w = k_new ? k_pool : nullptr;
    d.v_pool_w = k_new ? v_pool : nullptr;
    d.k_scale = k_scale;
    d.v_scale = v_scale;
    st = check_cuda(launch_decode(d, &plan->dec_inline, plan->decode_nt, stream),
                    "decode launch");
    if (st != RPA_OK) return st;
    MergeLaunch m{};
    m.rows = pl.rows;
    m.num_rows = plan->cap_rows;
    m.count = counts + 1;
    m.rows_per_item = d.rows_per_item;
    m.num_q_heads = s.num_q_heads;
    m.num_kv_heads = s.num_kv_heads;
    m.head_dim = s.head_dim;
    m.part_o = d.part_o;
    m.part_lse = d.part_lse;
    m.out = d.out;
    m.lse = lse;
    st = check_cuda(launch_merge(m, &plan->merge_inline, stream), "merge launch");
    if (st != RPA_OK) return st;
    st = check_cuda(cudaEventRecord(plan->join_ev, pf_stream), "join record");
    if (st != RPA_OK) return st;
    return check_cuda(cudaStreamWaitEvent(stream, plan->join_ev, 0), "join wait");
  }

  // A mixed batch runs the tensor-core kernel on the library's side stream, concurrently with
  // the split-KV decode kernel on the caller's stream: the decode CTAs fill the SMs that the
  // long prefill CTAs leave free.  The caller's stream waits for both before it goes on.
  const bool fork = !plan->pf_tiles.empty() && !plan->dec_items.empty();
  cudaStream_t pf_stream = stream;
  if (fork) {
    st = check_cuda(side_stream(stream, &pf_stream), "side stream");
    if (st != RPA_OK) return st;
    if (!plan->fork_ev) {
      st = check_cuda(cudaEventCreateWithFlags(&plan->fork_ev, cudaEventDisableTiming),
                      "event create");
      if (st != RPA_OK) return st;
      st = check_cuda(cudaEventCreateWithFlags(&plan->join_ev, cudaEventDisableTiming),
                      "event create");
      if (st != RPA_OK) return st;
    }
    st = check_cuda(cudaEventRecord(plan->fork_ev, stream), "fork record");
    if (st != RPA_OK) return st;
    st = check_cuda(cudaStreamWaitEvent(pf_stream, plan->fork_ev, 0), "fork wait");
    if (st != RPA_OK) return st;
  }

  if (!plan->pf_tiles.empty()) {
    PrefillLaunch p{};
    p.tiles = plan->inline_lists ? nullptr : reinterpret_cast<const PrefillTile*>(ws + plan->off_pf);
    p.num_tiles = (int32_t)plan->pf_tiles.size();
    p.q = static_cast<const uint16_t*>(q);
    p.num_tokens = s.num_tokens;
    p.num_q_heads = s.num_q_heads;
    p.num_kv_heads = s.num_kv_heads;
    p.head_dim = s.head_dim;
    p.causal = s.causal;
    p.scale_log2 = scale_log2;
    p.out = static_cast<uint16_t*>(out);
    p.lse = lse;
    p.persistent = fork ? 0 : 1;  // beside the decode kernel: one CTA per unit
    if (fork && plan->mixed_grid > 0) {
      // the planned split (mixed_grid): a persistent grid on part of the SMs, the decode kernel
      // launched once it is resident.  Not under stream capture, which the launch-completion
      // event is not meant for: there the unit-per-CTA launch stays.
      cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
      st = check_cuda(cudaStreamIsCapturing(stream, &cap), "capture status");
      if (st != RPA_OK) return st;
      if (cap == cudaStreamCaptureStatusNone) {
        if (!plan->launched_ev) {
          st = check_cuda(cudaEventCreateWithFlags(&plan->launched_ev, cudaEventDisableTiming),
                          "event create");
          if (st != RPA_OK) return st;
        }
        p.persistent = 1;
        p.max_ctas = plan->mixed_grid;
        p.launched = plan->launched_ev;
      }
    }
    if (plan->opts.sparse == 2) {
      p.qtile_table = group_table;
      p.qtile_count = group_count;
      p.qtiles_per_seq = plan->qtiles_per_seq;
    } else {
      p.group_table = group_table;
      p.group_count = group_count;
    }
    p.err = err;
    p.kv = kv;
    if (fuse_pf) {
      p.k_new = static_cast<const uint16_t*>(k_new);
      p.v_new = static_cast<const uint16_t*>(v_new);
      p.k_pool_w = k_pool;
      p.v_pool_w = v_pool;
      p.fuse_rows = fuse_box;
    }
    if (kv8) {
      // the codes are read in place and converted inside the kernel
      p.k_scale = k_scale;
      p.v_scale = v_scale;
    }
    st = check_cuda(launch_prefill(p, &plan->pf_inline, pf_stream), "prefill launch");
    if (st != RPA_OK) return st;
    if (p.launched) {
      st = check_cuda(cudaStreamWaitEvent(stream, p.launched, 0), "launch wait");
      if (st != RPA_OK) return st;
    }
  }
  if (!plan->dec_items.empty()) {
    DecodeLaunch d{};
    d.items = plan->inline_lists ? nullptr : reinterpret_cast<const DecodeItem*>(ws + plan->off_dec);
    d.num_items = (int32_t)plan->dec_items.size();
    d.rows_per_item = 8 * plan->decode_nt;
    d.q = static_cast<const uint16_t*>(q);
    d.num_q_heads = s.num_q_heads;
    d.num_kv_heads = s.num_kv_heads;
    d.head_dim = s.head_dim;
    d.causal = s.causal;
    d.scale_log2 = scale_log2;
    d.out = static_cast<uint16_t*>(out);
    d.lse = lse;
    d.part_o = reinterpret_cast<float*>(ws + plan->off_part_o);
    d.part_lse = reinterpret_cast<float*>(ws + plan->off_part_lse);
    d.err = err;
    d.kv = kv;
    const bool fused = k_new && (plan->fuse_write || fuse_pf);
    d.k_new = fused ? static_cast<const uint16_t*>(k_new) : nullptr;
    d.v_new = fused ? static_cast<const uint16_t*>(v_new) : nullptr;
    d.k_pool_w = fused ? k_pool : nullptr;
    d.v_pool_w = fused ? v_pool : nullptr;
    d.k_scale = k_scale;
    d.v_scale = v_scale;
    d.test_wait_ns = (uint32_t)plan->opts.wait_test_us * 1000u;
    st = check_cuda(launch_decode(d, &plan->dec_inline, plan->decode_nt, stream), "decode launch");
    if (st != RPA_OK) return st;
    if (!plan->merge_rows.empty()) {
      MergeLaunch m{};
      m.rows = plan->inline_lists ? nullptr : reinterpret_cast<const MergeRow*>(ws + plan->off_merge);
      m.num_rows = (int32_t)plan->merge_rows.size();
      m.rows_per_item = d.rows_per_item;
      m.num_q_heads = s.num_q_heads;
      m.num_kv_heads = s.num_kv_heads;
      m.head_dim = s.head_dim;
      m.part_o = d.part_o;
      m.part_lse = d.part_lse;
      m.out = d.out;
      m.lse = lse;
      st = check_cuda(launch_merge(m, &plan->merge_inline, stream), "merge launch");
      if (st != RPA_OK) return st;
    }
  }
  if (fork) {
    st = check_cuda(cudaEventRecord(plan->join_ev, pf_stream), "join record");
    if (st != RPA_OK) return st;
    st = check_cuda(cudaStreamWaitEvent(stream, plan->join_ev, 0), "join wait");
    if (st != RPA_OK) return st;
  }
  return RPA_OK;
}

rpa_status rpa_forward(rpa_plan_t plan, const void* q, const void* k_new, const void* v_new,
                       void* k_pool, void* v_pool, const int32_t* block_table,
                       const int32_t* cu_seqlens_q, const int32_t* seq_lens_k,
                       const int32_t* group_table, const int32_t* group_count, float scale,
                       void* out, float* lse, void* workspace, size_t workspace_bytes,
                       void* stream) {
  g_last_error.clear();
  return forward_impl(plan, q, k_new, v_new, k_pool, v_pool, block_table, cu_seqlens_q,
                      seq_lens_k, group_table, group_count, scale, out, lse, workspace,
                      workspace_bytes, stream, false, nullptr, nullptr);
}

rpa_status rpa_forward_kv8(rpa_plan_t plan, const void* q, const void* k_new, const void* v_new,
                           void* k_pool, void* v_pool, const float* k_scale,
                           const float* v_scale, const int32_t* block_table,
                           const int32_t* cu_seqlens_q, const int32_t* seq_lens_k,
                           const int32_t* group_table, const int32_t* group_count, float scale,
                           void* out, float* lse, void* workspace, size_t workspace_bytes,
                           void* stream) {
  g_last_error.clear();
  if (!plan) RPA_FAIL(RPA_ERR_INVALID_ARG, "plan is NULL");
  if (plan->shape.head_dim != 128)
    RPA_FAIL(RPA_ERR_UNSUPPORTED, "e4m3 pools need head_dim 128 (got %d)",
             plan->shape.head_dim);
  if (plan->device_mode && !plan->opts.kv_e4m3)
    RPA_FAIL(RPA_ERR_UNSUPPORTED,
             "e4m3 pools with a device plan need a plan made with opts.kv_e4m3 = 1");
  if (!plan->device_mode && !plan->pf_tiles.empty() && !plan->opts.kv_e4m3)
    RPA_FAIL(RPA_ERR_UNSUPPORTED,
             "e4m3 pools with rows for the tensor-core kernel need a plan made with "
             "opts.kv_e4m3 = 1");
  if (!k_scale || !v_scale) RPA_FAIL(RPA_ERR_INVALID_ARG, "k_scale and v_scale are required");
  if ((reinterpret_cast<uintptr_t>(k_scale) & 3u) || (reinterpret_cast<uintptr_t>(v_scale) & 3u))
    RPA_FAIL(RPA_ERR_INVALID_ARG, "k_scale / v_scale must be 4-byte aligned");
  return forward_impl(plan, q, k_new, v_new, k_pool, v_pool, block_table, cu_seqlens_q,
                      seq_lens_k, group_table, group_count, scale, out, lse, workspace,
                      workspace_bytes, stream, true, k_scale, v_scale);
}

rpa_status rpa_build_group_tables(const uint8_t* mask, int32_t num_seqs, int32_t num_q_heads,
                                  int32_t num_kv_heads, int32_t num_q_blocks,
                                  int32_t num_kv_blocks, int32_t* table, int32_t* count,
                                  void* stream) {
  g_last_error.clear();
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_blocks < 0 ||
      num_kv_blocks < 0)
    RPA_FAIL(RPA_ERR_SHAPE, "invalid table-builder sizes");
  if (num_q_heads % num_kv_heads != 0)
    RPA_FAIL(RPA_ERR_SHAPE, "num_q_heads (%d) must be a multiple of num_kv_heads (%d)",
             num_q_heads, num_kv_heads);
  if (num_kv_blocks > 65536) RPA_FAIL(RPA_ERR_UNSUPPORTED, "num_kv_blocks > 65536");
  if (num_seqs == 0) return RPA_OK;
  if (!table || !count || (!mask && num_q_blocks > 0 && num_kv_blocks > 0))
    RPA_FAIL(RPA_ERR_INVALID_ARG, "mask, table and count are required");
  return check_cuda(launch_group_tables(mask, num_seqs, num_q_heads, num_kv_heads, num_q_blocks,
                                        num_kv_blocks, table, count,
                                        static_cast<cudaStream_t>(stream)),
                    "group-table launch");
}

rpa_status rpa_build_qtile_tables(const uint8_t* mask, int32_t num_seqs, int32_t num_q_heads,
                                  int32_t num_q_blocks, int32_t num_kv_blocks,
                                  int32_t q_block_rows, int32_t* table, int32_t* count,
                                  void* stream) {
  g_last_error.clear();
  if (num_seqs < 0 || num_q_heads <= 0 || num_q_blocks < 0 || num_kv_blocks < 0)
    RPA_FAIL(RPA_ERR_SHAPE, "invalid table-builder sizes");
  if (q_block_rows <= 0 || q_block_rows > kPrefillTileRows ||
      kPrefillTileRows % q_block_rows != 0)
    RPA_FAIL(RPA_ERR_UNSUPPORTED, "q_block_rows %d must divide %d", q_block_rows,
             kPrefillTileRows);
  if (num_kv_blocks > 65536) RPA_FAIL(RPA_ERR_UNSUPPORTED, "num_kv_blocks > 65536");
  const int qb_per_tile = kPrefillTileRows / q_block_rows;
  const int ntiles = (num_q_blocks + qb_per_tile - 1) / qb_per_tile;
  if (num_seqs == 0 || ntiles == 0) return RPA_OK;
  if (!table || !count || (!mask && num_kv_blocks > 0))
    RPA_FAIL(RPA_ERR_INVALID_ARG, "mask, table and count are required");
  return check_cuda(launch_qtile_tables(mask, num_seqs, num_q_heads, num_q_blocks, num_kv_blocks,
                                        qb_per_tile, ntiles, table, count,
                                        static_cast<cudaStream_t>(stream)),
                    "query-tile table launch");
}

rpa_status rpa_device_error(int32_t* code, int32_t clear) {
  g_last_error.clear();
  if (!code) RPA_FAIL(RPA_ERR_INVALID_ARG, "code must not be NULL");
  int* err = nullptr;
  rpa_status st = check_cuda(device_error_word(&err), "device error word");
  if (st != RPA_OK) return st;
  st = check_cuda(cudaDeviceSynchronize(), "synchronize");
  if (st != RPA_OK) return st;
  int v = 0;
  st = check_cuda(cudaMemcpy(&v, err, sizeof(int), cudaMemcpyDeviceToHost), "read error word");
  if (st != RPA_OK) return st;
  *code = v;
  if (clear && v != 0) {
    const int zero = 0;
    st = check_cuda(cudaMemcpy(err, &zero, sizeof(int), cudaMemcpyHostToDevice),
                    "clear error word");
    if (st != RPA_OK) return st;
  }
  return v == 0 ? RPA_OK : RPA_ERR_DEVICE_CHECK;
}

}  // extern "C"
