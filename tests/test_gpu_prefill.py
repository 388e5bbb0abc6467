"""GPU parity of the tensor-core (tcgen05/TMEM) paged prefill path, the mixed batches and the
sparse block-union mode against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

from oracle import rpa_oracle as orc
from ragged_paged_attention_forward_b200 import api
from ragged_paged_attention_forward_b200 import workloads as wl
from tests.rpa_testing import (assert_close, assert_lse_close, oracle_forward, plan_for,
                                run_forward, to_device)

pytestmark = pytest.mark.gpu


def _sample_rows(batch, n, seed):
    g = np.random.default_rng(seed)
    T, Hq = batch.num_tokens, batch.num_q_heads
    rows = {(int(t), int(h)) for t, h in zip(g.integers(0, T, n), g.integers(0, Hq, n))}
    # always include each sequence's first and last token
    cu = batch.cu_seqlens_q.tolist()
    for b in range(batch.num_seqs):
        if cu[b + 1] > cu[b]:
            rows.add((cu[b], int(g.integers(0, Hq))))
            rows.add((cu[b + 1] - 1, int(g.integers(0, Hq))))
    return sorted(rows)


def _unit_rows(batch, units):
    """Every row of whole tensor-core work units.  A unit is a 128-query tile of one sequence
    and a pair of query heads of one KV group: ``(seq, local tile, first head)`` selects the
    tile's rows (clipped to the sequence) for heads ``h0`` and ``h0 + 1``."""
    cu = batch.cu_seqlens_q.tolist()
    rows = set()
    for b, tile, h0 in units:
        lo, hi = tile * 128, min(cu[b + 1] - cu[b], tile * 128 + 128)
        assert lo < hi, (b, tile)
        rows.update((cu[b] + i, h) for i in range(lo, hi) for h in (h0, h0 + 1))
    return sorted(rows)


def test_prefill_small_no_past():
    b = wl.ragged_batch([200, 64], [200, 64], 8, 2, 128, 64, seed=51)
    ref, ref_lse, kp, vp = oracle_forward(b)
    out, lse, gk, gv, plan = run_forward(b)
    assert plan.info().batch_class == api.CLASS_PREFILL
    assert_close(out, ref)
    assert_lse_close(lse, ref_lse)
    assert np.array_equal(orc.bits16(gk), kp) and np.array_equal(orc.bits16(gv), vp)


@pytest.mark.parametrize("layout", [wl.SEQ_MAJOR, wl.HEAD_MAJOR])
@pytest.mark.parametrize("page", [16, 32, 64, 128, 256])
def test_chunked_prefill_with_past(page, layout):
    # pasts 300, 130 and 743, every row on the tensor-core kernel: the scatter kernel writes
    # the new K/V first; the whole pool is compared bit for bit
    b = wl.ragged_batch([430, 170, 1000], [130, 40, 257], 8, 2, 128, page, seed=52 + page,
                        layout=layout)
    ref, ref_lse, kp, vp = oracle_forward(b)
    out, lse, gk, gv, plan = run_forward(b)
    info = plan.info()
    assert info.num_prefill_tiles > 0
    assert info.launches_forward == 2      # scatter + tensor-core kernel
    assert_close(out, ref)
    assert_lse_close(lse, ref_lse)
    assert np.array_equal(orc.bits16(gk), kp) and np.array_equal(orc.bits16(gv), vp)


@pytest.mark.parametrize("straddle", [False, True])
@pytest.mark.parametrize("page", [16, 64, 256])
def test_fused_write_equals_separate_write(page, straddle):
    # A mixed batch: both attention kernels write their rows' new K/V themselves (the
    # tensor-core kernel reads its rows' new keys from k_new / v_new).  Against rpa_write_kv
    # followed by an rpa_forward without new rows: same pools, same outputs bit for bit.  The
    # chunks' pasts (256, 0, 512) are box-aligned, so no scatter kernel runs in the fused step;
    # with a past of 33 the first new rows share a box with older keys and are scattered first.
    kv = [400, 333 if straddle else 300, 1000, 700]
    b = wl.ragged_batch(kv, [144, 300, 488, 1], 8, 2, 128, page, seed=59 + page)
    plan = plan_for(b)
    info = plan.info()
    assert info.batch_class == api.CLASS_MIXED
    assert info.launches_forward == (4 if straddle else 3)  # [scatter,] tensor-core, decode, merge
    fused = run_forward(b)
    split = run_forward(b, fused=False)
    assert torch.equal(fused[0], split[0]) and torch.equal(fused[1], split[1])
    # the pools hold NaN in their free slots: compare bit patterns
    assert np.array_equal(orc.bits16(fused[2]), orc.bits16(split[2]))
    assert np.array_equal(orc.bits16(fused[3]), orc.bits16(split[3]))
    ref, _, kp, vp = oracle_forward(b)
    assert_close(fused[0], ref)
    assert np.array_equal(orc.bits16(fused[2]), kp) and np.array_equal(orc.bits16(fused[3]), vp)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (8, 1)])
def test_prefill_heads_and_dims(D, Hq, Hkv):
    b = wl.ragged_batch([300, 129], [150, 129], Hq, Hkv, D, 16, seed=53 + D + Hq)
    ref, ref_lse, _, _ = oracle_forward(b)
    out, lse, _, _, _ = run_forward(b)
    assert_close(out, ref)
    assert_lse_close(lse, ref_lse)


def test_varlen_regression_case_forced_on_tensor_cores():
    # B=2, q_lens (32, 16), head size 128, MHA (the fused varlen prefill regression shape of
    # the WebGPU page's test list) -- every row through the tensor-core kernel
    b = wl.ragged_batch([32, 16], [32, 16], 4, 4, 128, 16, seed=54)
    ref, ref_lse, _, _ = oracle_forward(b)
    out, lse, _, _, plan = run_forward(b, plan_opts=dict(force_class=api.CLASS_PREFILL))
    assert plan.info().num_decode_items == 0
    assert_close(out, ref)
    assert_lse_close(lse, ref_lse)


@pytest.mark.parametrize("causal", [True, False])
def test_mixed_q_len_with_past(causal):
    # the failing WebGPU case: mixed q_len with past > 0
    b = wl.ragged_batch([16, 40, 300, 77, 1000], [16, 4, 300, 1, 33], 4, 2, 128, 16, seed=55,
                        causal=causal)
    ref, ref_lse, kp, vp = oracle_forward(b)
    out, lse, gk, gv, plan = run_forward(b)
    info = plan.info()
    assert info.batch_class == api.CLASS_MIXED
    assert info.num_prefill_tiles > 0 and info.num_decode_items > 0
    assert_close(out, ref)
    assert_lse_close(lse, ref_lse)
    assert np.array_equal(orc.bits16(gk), kp) and np.array_equal(orc.bits16(gv), vp)
    forced = run_forward(b, plan_opts=dict(force_class=api.CLASS_PREFILL))
    assert_close(forced[0], ref)
    assert np.array_equal(orc.bits16(forced[2]), kp) and np.array_equal(orc.bits16(forced[3]), vp)


@pytest.mark.parametrize("scale", [0.0, 0.02, -0.09])
def test_prefill_explicit_scale(scale):
    b = wl.ragged_batch([260], [200], 4, 2, 64, 64, seed=56)
    ref, ref_lse, _, _ = oracle_forward(b, scale=scale)
    out, lse, _, _, _ = run_forward(b, scale=scale)
    assert_close(out, ref)
    assert_lse_close(lse, ref_lse)


def test_prefill_head_major_equals_seq_major():
    b = wl.ragged_batch([333, 128], [200, 128], 8, 2, 128, 64, seed=57)
    o1 = run_forward(b)[0]
    o2 = run_forward(wl.to_head_major(b))[0]
    ref, _, _, _ = oracle_forward(b)
    assert_close(o1, ref)
    assert_close(o2, ref)


@pytest.mark.parametrize("scale", [0.5, 2.0, 50.0])
def test_prefill_large_scores_move_the_reference_max(scale):
    # Large softmax scales make later key tiles beat the first tile's row max by far more
    # than 64 in log2 units, so tiles are redone against their own max with O rescaled.
    # Sharp attention puts single V rows into the output, so the rounding bound scales with
    # max|V|: P and the output are each rounded to bf16 (relative error <= 2^-8), giving
    # |err| <= 2 * 2^-8 * max|V| plus fp32 noise.
    b = wl.ragged_batch([1500, 700], [900, 700], 8, 2, 128, 64, seed=61)
    ref, ref_lse, _, _ = oracle_forward(b, scale=scale)
    out, lse, _, _, _ = run_forward(b, scale=scale)
    assert torch.isfinite(out.float()).all()
    vmax = max(float(v.float().abs().max()) for v in b.v_logical)
    assert_close(out, ref, tol_max=2.0 * 2.0 ** -8 * vmax + 1e-3)
    assert_lse_close(lse, ref_lse)


@pytest.mark.parametrize("D", [64, 128])
def test_prefill_output_only_16_byte_aligned(D):
    # The epilogue writes 32 bytes per store when the output is 32-byte aligned and 16 bytes
    # otherwise; an output 16 bytes past an aligned base takes the narrow stores and must
    # give the same bits.
    b = wl.ragged_batch([700, 300], [500, 300], 8, 2, D, 64, seed=59)
    plan = plan_for(b)
    d = to_device(b)
    T, Hq = b.num_tokens, b.num_q_heads
    ws = torch.empty(max(plan.workspace_bytes, 256), dtype=torch.uint8, device="cuda")
    outs = []
    for shift in (0, 8):  # elements: 0 and 16 bytes
        base = torch.full((T * Hq * D + 16,), float("nan"), dtype=torch.bfloat16, device="cuda")
        out = base[shift:shift + T * Hq * D].view(T, Hq, D)
        assert (out.data_ptr() % 32 == 0) == (shift == 0)
        api.rpa_forward(plan, d["q"], d["k_new"], d["v_new"], d["k_pool"], d["v_pool"],
                        d["block_table"], d["cu_seqlens_q"], d["seq_lens_k"], None, None,
                        b.scale, out, None, ws)
        torch.cuda.synchronize()
        assert api.rpa_device_error(clear=True) == 0
        outs.append(out.cpu())
    assert plan.info().num_prefill_tiles > 0
    assert torch.equal(outs[0], outs[1])
    ref, _, _, _ = oracle_forward(b)
    assert_close(outs[1], ref)


def test_prefill_page_permutation_gives_identical_output():
    b = wl.ragged_batch([500, 260], [300, 260], 8, 2, 128, 16, seed=58)
    o1 = run_forward(b)[0]
    o2 = run_forward(wl.permute_pages(b, seed=3))[0]
    assert torch.equal(o1, o2)


def test_prefill_config_full_size_whole_units():
    # The prefill workload (4 x 4096 causal) in the launch the benchmark times: a persistent
    # grid of one CTA per SM walking 2048 units (128-query tile x query-head pair) in rounds
    # of the grid size, left to right, then right to left.  The planner sorts tiles heaviest
    # first (stable), so list position p holds sequence p % 4, tile 31 - p // 4, and unit
    # 16 p + pair.  Whole units are compared: the first, a middle and the last tile of every
    # sequence, and units of the walk's first round (positions 0, 5) and second round
    # (positions 9 and 13, pairs 8 and 3: units 152 and 211).
    b = wl.prefill()
    out, lse, gk, gv, plan = run_forward(b)
    assert plan.info().batch_class == api.CLASS_PREFILL
    units = [(s, 0, 2 * s) for s in range(4)] + [(s, 15, 8 + 2 * s) for s in range(4)] + \
            [(s, 31, 16 + 2 * s) for s in range(4)] + \
            [(0, 31, 0), (1, 30, 14), (1, 29, 16), (1, 28, 6)]
    rows = _unit_rows(b, units)
    ref, ref_lse, kp, vp = oracle_forward(b, rows=rows)
    assert_close(out, ref, rows=rows)
    assert_lse_close(lse, ref_lse, rows=rows)
    assert np.array_equal(orc.bits16(gk), kp) and np.array_equal(orc.bits16(gv), vp)
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("shuffle", [False, True])
def test_mixed_config_full_size_whole_units(shuffle):
    # The mixed workload: 48 decode rows (split-KV kernel) and chunks of 512 and 976 queries
    # with past 1024 and 8192 (tensor-core kernel, one CTA per unit).  Whole units of both
    # chunks -- first, middle and last tile, the 976-query chunk's last tile ragged (80 rows)
    # -- and every query head of each decode row's KV group.
    b = wl.mixed(shuffle=shuffle)
    out, lse, _, _, plan = run_forward(b)
    info = plan.info()
    assert info.num_prefill_tiles > 0 and info.num_decode_items > 0
    cu = b.cu_seqlens_q.tolist()
    q_lens = [cu[i + 1] - cu[i] for i in range(b.num_seqs)]
    c512, c976 = q_lens.index(512), q_lens.index(976)
    units = [(c512, 0, 0), (c512, 1, 30), (c512, 3, 12),
             (c976, 0, 4), (c976, 4, 18), (c976, 7, 0), (c976, 7, 26)]
    rows = set(_unit_rows(b, units))
    for i in range(b.num_seqs):
        if q_lens[i] == 1:
            g = i % 8
            rows.update((cu[i], h) for h in range(4 * g, 4 * g + 4))
    rows = sorted(rows)
    ref, ref_lse, _, _ = oracle_forward(b, rows=rows)
    assert_close(out, ref, rows=rows)
    assert_lse_close(lse, ref_lse, rows=rows)
    assert torch.isfinite(out.float()).all()


def test_mixed_output_is_stream_ordered():
    # The tensor-core kernel runs on the library's side stream beside the decode kernel: work
    # queued on the caller's stream right after the call must see every output row.
    b = wl.ragged_batch([700, 3000, 1500, 40], [300, 1, 1, 40], 8, 2, 128, 16, seed=62)
    plan = plan_for(b)
    assert plan.info().batch_class == api.CLASS_MIXED
    d = to_device(b)
    out = torch.full_like(d["q"], float("nan"))
    ws = torch.empty(max(plan.workspace_bytes, 256), dtype=torch.uint8, device="cuda")
    api.rpa_forward(plan, d["q"], d["k_new"], d["v_new"], d["k_pool"], d["v_pool"],
                    d["block_table"], d["cu_seqlens_q"], d["seq_lens_k"], None, None, b.scale,
                    out, None, ws)
    snap = out.clone()  # queued on the same stream, no synchronisation in between
    torch.cuda.synchronize()
    assert api.rpa_device_error(clear=True) == 0
    assert torch.equal(snap, out)
    ref, _, _, _ = oracle_forward(b)
    assert_close(out.cpu(), ref)


def test_split_mixed_step_is_stream_ordered():
    # The mixed workload plans a split: a persistent tensor-core grid on part of the SMs and
    # the decode kernel, launched once that grid is resident, on the rest.  Work queued on the
    # caller's stream right after the call must see every output row, and the rows must be
    # right: every decode row's KV group and a whole unit of each chunk.
    b = wl.mixed()
    plan = plan_for(b)
    info = plan.info()
    assert 0 < info.tensor_core_grid < 148
    d = to_device(b)
    out = torch.full_like(d["q"], float("nan"))
    ws = torch.empty(max(plan.workspace_bytes, 256), dtype=torch.uint8, device="cuda")
    api.rpa_forward(plan, d["q"], d["k_new"], d["v_new"], d["k_pool"], d["v_pool"],
                    d["block_table"], d["cu_seqlens_q"], d["seq_lens_k"], None, None, b.scale,
                    out, None, ws)
    snap = out.clone()  # queued on the same stream, no synchronisation in between
    torch.cuda.synchronize()
    assert api.rpa_device_error(clear=True) == 0
    assert torch.equal(snap, out)
    cu = b.cu_seqlens_q.tolist()
    q_lens = [cu[i + 1] - cu[i] for i in range(b.num_seqs)]
    rows = set(_unit_rows(b, [(q_lens.index(512), 2, 6), (q_lens.index(976), 5, 20)]))
    for i in range(b.num_seqs):
        if q_lens[i] == 1:
            rows.update((cu[i], h) for h in range(4 * (i % 8), 4 * (i % 8) + 4))
    rows = sorted(rows)
    ref, _, kp, _ = oracle_forward(b, rows=rows)
    assert_close(out.cpu(), ref, rows=rows)
    assert np.array_equal(orc.bits16(d["k_pool"].cpu()), kp)


def test_mixed_steps_from_two_caller_streams():
    # Two callers on two streams of one device: each mixed step forks its tensor-core kernel
    # onto a side stream that belongs to its own caller stream and joins it back, so work
    # queued on each caller's stream right after its call sees every output row.
    b1 = wl.ragged_batch([700, 3000, 1500, 40], [300, 1, 1, 40], 8, 2, 128, 16, seed=62)
    b2 = wl.ragged_batch([900, 2000, 64], [200, 1, 64], 8, 2, 128, 16, seed=63)
    runs = []
    for b in (b1, b2):
        plan = plan_for(b)
        assert plan.info().batch_class == api.CLASS_MIXED
        d = to_device(b)
        out = torch.full_like(d["q"], float("nan"))
        ws = torch.empty(max(plan.workspace_bytes, 256), dtype=torch.uint8, device="cuda")
        runs.append((b, plan, d, out, ws, torch.cuda.Stream(), torch.empty_like(out)))
    torch.cuda.synchronize()
    for b, plan, d, out, ws, s, snap in runs:
        api.rpa_forward(plan, d["q"], d["k_new"], d["v_new"], d["k_pool"], d["v_pool"],
                        d["block_table"], d["cu_seqlens_q"], d["seq_lens_k"], None, None,
                        b.scale, out, None, ws, stream=s)
        with torch.cuda.stream(s):
            snap.copy_(out)  # queued on the caller's stream, no synchronisation in between
    torch.cuda.synchronize()
    assert api.rpa_device_error(clear=True) == 0
    for b, plan, d, out, ws, s, snap in runs:
        assert torch.equal(snap, out)
        ref, _, kp, vp = oracle_forward(b)
        assert_close(out.cpu(), ref)
        assert np.array_equal(orc.bits16(d["k_pool"].cpu()), kp)


# ------------------------------------------------------------------ sparse block-union mode

def _sparse_case(kv_len, chunk, page, seed, density=None, Hq=8, Hkv=2, D=128):
    b = wl.ragged_batch([kv_len], [chunk], Hq, Hkv, D, page, seed=seed, layout=wl.HEAD_MAJOR)
    nqb = -(-chunk // page)
    nkb = b.max_blocks
    if density is None:
        mask = wl.structured_block_mask(1, Hq, Hkv, nqb, nkb, seed=seed + 1,
                                        past_blocks=(kv_len - chunk) // page)
    else:
        mask = wl.iid_block_mask(1, Hq, nqb, nkb, seed=seed + 1, density=density)
    table, count = orc.build_group_tables(mask, Hkv)
    return b, torch.from_numpy(table), torch.from_numpy(count)


@pytest.mark.parametrize("page", [16, 64, 128])
def test_sparse_small(page):
    b, table, count = _sparse_case(1500, 300, page, seed=60 + page)
    ref, ref_lse, kp, vp = oracle_forward(b, group_table=table.numpy(),
                                          group_count=count.numpy())
    out, lse, gk, gv, plan = run_forward(b, group_table=table, group_count=count)
    assert plan.info().num_decode_items == 0
    assert_close(out, ref)
    assert_lse_close(lse, ref_lse)
    assert np.array_equal(orc.bits16(gk), kp) and np.array_equal(orc.bits16(gv), vp)


def test_sparse_all_ones_equals_dense():
    b, table, count = _sparse_case(900, 200, 64, seed=61, density=1.0)
    dense = run_forward(b)[0]
    sp = run_forward(b, group_table=table, group_count=count)[0]
    ref, _, _, _ = oracle_forward(b)
    assert_close(dense, ref)
    assert_close(sp, ref)


def test_sparse_rows_without_visible_blocks():
    b = wl.ragged_batch([256], [256], 4, 1, 64, 64, seed=62, layout=wl.HEAD_MAJOR)
    mask = np.zeros((1, 4, 4, 4), dtype=np.uint8)
    mask[..., 2:] = 1             # rows before position 128 see nothing
    table, count = orc.build_group_tables(mask, 1)
    ref, ref_lse, _, _ = oracle_forward(b, group_table=table, group_count=count)
    out, lse, _, _, _ = run_forward(b, group_table=torch.from_numpy(table),
                                    group_count=torch.from_numpy(count))
    assert torch.all(out[:128] == 0)
    assert torch.all(torch.isneginf(lse[:128]))
    assert_close(out, ref)
    assert_lse_close(lse, ref_lse)


def test_sparse_config_full_size_whole_units():
    # The sparse workload (2048 queries at 128K context, per-group tables) in the persistent
    # launch: 16 tiles x 16 pairs = 256 units over 148 CTAs.  The list holds tile 15 - p at
    # position p, unit 16 p + pair.  Whole units: the first of round one (tile 15, pair 0),
    # a middle one (tile 8, pair 9), and two of round two (tile 6, pair 6 = unit 150; tile 0,
    # pair 15 = unit 255, the last).
    b, mask = wl.sparse()
    m = mask.cuda()
    nkb = mask.shape[-1]
    table = torch.empty(1, 8, nkb, dtype=torch.int32, device="cuda")
    count = torch.empty(1, 8, dtype=torch.int32, device="cuda")
    api.rpa_build_group_tables(m, 8, table, count)
    torch.cuda.synchronize()
    rt, rc = orc.build_group_tables(mask, 8)
    assert np.array_equal(table.cpu().numpy(), rt) and np.array_equal(count.cpu().numpy(), rc)
    out, lse, _, _, _ = run_forward(b, group_table=table, group_count=count)
    rows = _unit_rows(b, [(0, 15, 0), (0, 8, 18), (0, 6, 12), (0, 0, 30)])
    ref, ref_lse, _, _ = oracle_forward(b, group_table=rt, group_count=rc, rows=rows)
    assert_close(out, ref, rows=rows)
    assert_lse_close(lse, ref_lse, rows=rows)


def test_sparse_persistent_walk_with_empty_units():
    # 16 query tiles x 16 head pairs = 256 units over at most one CTA per SM, so CTAs walk
    # several units.  The heads of KV groups 4-7 select only blocks from position 3072 on, so
    # for them the first 8 tiles (rows before position 3072) have no key tile at all: those
    # units produce zeros and lse = -inf, and come after units with work in a CTA's walk.
    b = wl.ragged_batch([4096], [2048], 32, 8, 128, 64, seed=71, layout=wl.HEAD_MAJOR)
    nqb, nkb = 2048 // 64, b.max_blocks
    rng = np.random.default_rng(72)
    mask = (rng.random((1, 32, nqb, nkb)) < 0.3).astype(np.uint8)
    mask[..., 4096 // 64:] = 0     # no block past the sequence
    mask[:, 16:, :, :48] = 0       # groups 4-7: blocks 48.. only (keys 3072..)
    table, count = orc.build_group_tables(mask, 8)
    out, lse, _, _, _ = run_forward(b, group_table=torch.from_numpy(table),
                                    group_count=torch.from_numpy(count))
    assert torch.all(out[:1024, 16:] == 0)
    assert torch.all(torch.isneginf(lse[:1024, 16:]))
    # whole units, in list order (tile 15 - p at position p, unit 16 p + pair): round one
    # with keys (tile 15, pair 8) and without (tile 7, pair 12 = unit 140); round two
    # without keys (tile 6, pair 9 = unit 153) and with (tile 5, pair 2; tile 0, pair 0)
    rows = sorted(set(_sample_rows(b, 24, seed=73)) |
                  set(_unit_rows(b, [(0, 15, 16), (0, 7, 24), (0, 6, 18), (0, 5, 4),
                                     (0, 0, 0)])))
    ref, ref_lse, _, _ = oracle_forward(b, group_table=table, group_count=count, rows=rows)
    assert_close(out, ref, rows=rows)
    assert_lse_close(lse, ref_lse, rows=rows)


# ------------------------------------------------------------------ odd GQA group sizes

@pytest.mark.parametrize("layout", [wl.SEQ_MAJOR, wl.HEAD_MAJOR])
@pytest.mark.parametrize("Hq,Hkv", [(12, 4), (40, 8)])
def test_odd_group_size_mixed_batch(Hq, Hkv, layout):
    # G = 3 and G = 5 (the WebGPU page's test list covers MHA and GQA variants): the
    # tensor-core kernel then takes one query head per unit (a head pair must share a KV
    # group), and the split-KV kernel packs G x q_len query rows of a group into its MMA's N.
    b = wl.ragged_batch([1, 300, 777, 260, 2000], [1, 2, 1, 200, 150], Hq, Hkv, 128, 16,
                        seed=97 + Hq, layout=layout)
    ref, ref_lse, kp, vp = oracle_forward(b)
    out, lse, gk, gv, plan = run_forward(b)
    info = plan.info()
    assert info.num_decode_items > 0 and info.num_prefill_tiles > 0
    assert_close(out, ref)
    assert_lse_close(lse, ref_lse)
    assert np.array_equal(orc.bits16(gk), kp) and np.array_equal(orc.bits16(gv), vp)


@pytest.mark.parametrize("Hq,Hkv", [(12, 4), (40, 8)])
def test_odd_group_size_prefill_persistent(Hq, Hkv):
    # a prefill-only batch: the persistent grid walks one-head units
    b = wl.ragged_batch([700, 1300, 129], [700, 600, 129], Hq, Hkv, 128, 64, seed=99 + Hq)
    ref, ref_lse, kp, vp = oracle_forward(b)
    out, lse, gk, gv, plan = run_forward(b)
    assert plan.info().batch_class == api.CLASS_PREFILL
    assert_close(out, ref)
    assert_lse_close(lse, ref_lse)
    assert np.array_equal(orc.bits16(gk), kp) and np.array_equal(orc.bits16(gv), vp)


@pytest.mark.parametrize("Hq,Hkv", [(12, 4), (40, 8)])
def test_odd_group_size_decode(Hq, Hkv):
    b = wl.ragged_batch([1, 17, 300, 1025, 64], [1] * 5, Hq, Hkv, 128, 16, seed=101 + Hq)
    ref, ref_lse, kp, vp = oracle_forward(b)
    out, lse, gk, gv, plan = run_forward(b, plan_opts=dict(decode_split_keys=256))
    info = plan.info()
    assert info.batch_class == api.CLASS_DECODE and info.num_merge_rows > 0
    assert_close(out, ref)
    assert_lse_close(lse, ref_lse)
    assert np.array_equal(orc.bits16(gk), kp) and np.array_equal(orc.bits16(gv), vp)
