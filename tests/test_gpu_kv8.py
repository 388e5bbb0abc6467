"""GPU parity of the e4m3 (fp8) KV-cache path against the fp64 oracle: the split-KV decode
kernel and the tensor-core kernel, both reading the codes in place.

The quantising KV write must produce the oracle's codes bit for bit; attention over the
dequantised cache must match within the tolerance derived in tests.rpa_testing.  Runs through
the C ABI (rpa_forward_kv8)."""
import numpy as np
import pytest
import torch

from oracle import rpa_oracle as orc
from ragged_paged_attention_forward_b200 import api
from ragged_paged_attention_forward_b200 import workloads as wl
from tests.rpa_testing import assert_kv8_close, assert_lse_close, kv8_vmax, plan_for

pytestmark = pytest.mark.gpu


def run_kv8(b8, ks, vs, *, plan_opts=None, with_new=True, scale=None, group_table=None,
            group_count=None):
    plan = plan_for(b8, **(plan_opts or {}))
    d = {k: getattr(b8, k).cuda().contiguous() for k in (
        "q", "k_new", "v_new", "k_pool", "v_pool", "block_table", "cu_seqlens_q", "seq_lens_k")}
    T, Hq, D = b8.q.shape
    out = torch.full((T, Hq, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((T, Hq), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(max(plan.workspace_bytes, 256), dtype=torch.uint8, device="cuda")
    api.rpa_forward_kv8(plan, d["q"], d["k_new"] if with_new else None,
                        d["v_new"] if with_new else None, d["k_pool"], d["v_pool"],
                        ks.cuda(), vs.cuda(), d["block_table"], d["cu_seqlens_q"],
                        d["seq_lens_k"], b8.scale if scale is None else scale, out, lse, ws,
                        group_table=None if group_table is None else group_table.cuda(),
                        group_count=None if group_count is None else group_count.cuda())
    torch.cuda.synchronize()
    assert api.rpa_device_error(clear=True) == 0
    return out.cpu(), lse.cpu(), d["k_pool"].cpu(), d["v_pool"].cpu(), plan


def oracle_kv8(b8, ks, vs, with_new=True, scale=None, rows=None, **tables):
    return orc.forward_kv8(b8.q, b8.k_new if with_new else None, b8.v_new if with_new else None,
                           b8.k_pool, b8.v_pool, ks.numpy(), vs.numpy(), b8.block_table,
                           b8.cu_seqlens_q, b8.seq_lens_k,
                           scale=b8.scale if scale is None else scale, causal=b8.causal,
                           page_size=b8.page_size, layout=b8.layout, rows=rows, **tables)


def check_out(out, ref, vs, b8, v_pool_after, rows=None):
    # the bound of tests.rpa_testing.kv8_output_errors (derived there): pointwise
    # 2^-10 max|V| + 2^-8 |o| with max|V| what the written V pool holds, mean-abs <= 2e-3
    vmax = kv8_vmax(v_pool_after, vs.numpy(), b8.block_table, b8.layout)
    assert_kv8_close(out, ref, vmax, rows=rows)


@pytest.mark.parametrize("page", [16, 64])
@pytest.mark.parametrize("layout", [wl.SEQ_MAJOR, wl.HEAD_MAJOR])
def test_kv8_decode_write_and_attention(page, layout):
    b = wl.ragged_batch([1, 17, 300, 1025, 64], [1, 1, 1, 1, 1], 32, 8, 128, page, seed=900 + page)
    if layout == wl.HEAD_MAJOR:
        b = wl.to_head_major(b)
    b8, ks, vs = wl.with_kv8_pools(b, seed=901)
    out, lse, kp, vp, plan = run_kv8(b8, ks, vs)
    assert plan.info().num_prefill_tiles == 0
    ref, ref_lse, kp_ref, vp_ref = oracle_kv8(b8, ks, vs)
    assert np.array_equal(kp.numpy(), kp_ref) and np.array_equal(vp.numpy(), vp_ref)
    check_out(out, ref, vs, b8, vp_ref)
    assert_lse_close(lse, ref_lse)


@pytest.mark.parametrize("Hq,Hkv,q_len", [(32, 8, 1), (32, 8, 4), (64, 8, 1), (64, 4, 1),
                                          (8, 8, 1), (128, 8, 2)])
def test_kv8_group_sizes_and_short_queries(Hq, Hkv, q_len):
    b = wl.ragged_batch([q_len, 200, 777], [q_len] * 3, Hq, Hkv, 128, 16, seed=910 + Hq + q_len)
    b8, ks, vs = wl.with_kv8_pools(b, seed=911)
    # q_len > 1 makes the batch "mixed", whose decode rows stop at 16: 32 rows need the
    # decode class forced
    opts = dict(force_class=api.CLASS_DECODE) if q_len * (Hq // Hkv) > 16 else None
    out, lse, kp, vp, plan = run_kv8(b8, ks, vs, plan_opts=opts)
    assert plan.info().num_prefill_tiles == 0
    ref, ref_lse, kp_ref, vp_ref = oracle_kv8(b8, ks, vs)
    assert np.array_equal(kp.numpy(), kp_ref) and np.array_equal(vp.numpy(), vp_ref)
    check_out(out, ref, vs, b8, vp_ref)
    assert_lse_close(lse, ref_lse)


def test_kv8_split_keys_and_merge():
    b = wl.ragged_batch([5000, 3333, 129], [1, 1, 1], 32, 8, 128, 16, seed=920)
    b8, ks, vs = wl.with_kv8_pools(b, seed=921)
    out, lse, kp, vp, plan = run_kv8(b8, ks, vs, plan_opts=dict(decode_split_keys=512))
    assert plan.info().num_merge_rows > 0
    ref, ref_lse, kp_ref, vp_ref = oracle_kv8(b8, ks, vs)
    assert np.array_equal(kp.numpy(), kp_ref) and np.array_equal(vp.numpy(), vp_ref)
    check_out(out, ref, vs, b8, vp_ref)
    assert_lse_close(lse, ref_lse)


def test_kv8_without_new_tokens_reads_cache_only():
    b = wl.ragged_batch([40, 90], [1, 1], 16, 4, 128, 16, seed=930)
    b8, ks, vs = wl.with_kv8_pools(b, seed=931)
    # the new tokens' slots hold NaN codes: attention over them must not be asked for, so
    # write them first through a plain call and then attend with k_new = v_new = None
    _, _, kp, vp, _ = run_kv8(b8, ks, vs)
    import dataclasses
    b8w = dataclasses.replace(b8, k_pool=kp, v_pool=vp)
    out, lse, kp2, vp2, _ = run_kv8(b8w, ks, vs, with_new=False)
    ref, ref_lse, _, _ = oracle_kv8(b8w, ks, vs, with_new=False)
    assert np.array_equal(kp2.numpy(), kp.numpy())
    check_out(out, ref, vs, b8, vp)
    assert_lse_close(lse, ref_lse)


@pytest.mark.parametrize("layout", [wl.SEQ_MAJOR, wl.HEAD_MAJOR])
@pytest.mark.parametrize("page", [16, 64])
def test_kv8_mixed_batch_through_both_kernels(layout, page):
    # decode rows and prefill chunks (with past) both on the e4m3 pools, the tensor-core
    # kernel converting its tiles to f16 itself; the new tokens of both quantised by the
    # scatter kernel
    b = wl.ragged_batch([300, 40, 1500, 9, 700], [300, 1, 213, 1, 77], 32, 8, 128, page,
                        seed=960 + page)
    if layout == wl.HEAD_MAJOR:
        b = wl.to_head_major(b)
    b8, ks, vs = wl.with_kv8_pools(b, seed=961)
    out, lse, kp, vp, plan = run_kv8(b8, ks, vs, plan_opts=dict(kv_e4m3=True))
    info = plan.info()
    assert info.num_prefill_tiles > 0 and info.num_decode_items > 0
    ref, ref_lse, kp_ref, vp_ref = oracle_kv8(b8, ks, vs)
    assert np.array_equal(kp.numpy(), kp_ref) and np.array_equal(vp.numpy(), vp_ref)
    check_out(out, ref, vs, b8, vp_ref)
    assert_lse_close(lse, ref_lse)


def test_kv8_prefill_only_and_non_causal():
    import dataclasses
    b = wl.ragged_batch([640, 200], [512, 200], 16, 4, 128, 32, seed=970)
    for causal in (True, False):
        bc = dataclasses.replace(b, causal=causal)
        b8, ks, vs = wl.with_kv8_pools(bc, seed=971)
        out, lse, kp, vp, plan = run_kv8(b8, ks, vs, plan_opts=dict(kv_e4m3=True))
        assert plan.info().num_decode_items == 0
        ref, ref_lse, kp_ref, vp_ref = oracle_kv8(b8, ks, vs)
        assert np.array_equal(kp.numpy(), kp_ref) and np.array_equal(vp.numpy(), vp_ref)
        check_out(out, ref, vs, b8, vp_ref)
        assert_lse_close(lse, ref_lse)


def test_kv8_rejects_unsupported_plans():
    b = wl.ragged_batch([300, 40], [300, 1], 8, 2, 128, 16, seed=940)   # has a prefill row
    b8, ks, vs = wl.with_kv8_pools(b, seed=941)
    with pytest.raises(api.RPAError) as e:
        run_kv8(b8, ks, vs)
    assert "UNSUPPORTED" in str(e.value) or "decode" in str(e.value)
    b64 = wl.ragged_batch([30], [1], 8, 2, 64, 16, seed=942)
    b64_8, ks, vs = wl.with_kv8_pools(b64, seed=943)
    with pytest.raises(api.RPAError):
        run_kv8(b64_8, ks, vs)


def _sample_rows(batch, n, seed):
    g = np.random.default_rng(seed)
    T, Hq = batch.num_tokens, batch.num_q_heads
    rows = {(int(t), int(h)) for t, h in zip(g.integers(0, T, n), g.integers(0, Hq, n))}
    cu = batch.cu_seqlens_q.tolist()
    for b in range(batch.num_seqs):
        if cu[b + 1] > cu[b]:
            rows.add((cu[b], int(g.integers(0, Hq))))
            rows.add((cu[b + 1] - 1, int(g.integers(0, Hq))))
    return sorted(rows)


def _check_rows(out, lse, ref, ref_lse, rows, vs, b8, v_pool_after):
    check_out(out, ref, vs, b8, v_pool_after, rows=rows)
    for t, h in rows:
        assert abs(float(lse[t, h]) - ref_lse[t, h]) <= 2e-3, (t, h)


def test_kv8_decode_workload_full_size_sampled():
    # the benchmark's decode batch (64 sequences, kv 512-8192) over e4m3 pools, in the launch
    # configuration the benchmark times; the oracle computes sampled rows one by one
    b8, ks, vs = wl.with_kv8_pools(wl.decode(), seed=1234)
    out, lse, kp, vp, plan = run_kv8(b8, ks, vs)
    assert plan.info().batch_class == api.CLASS_DECODE
    rows = _sample_rows(b8, 48, seed=5)
    ref, ref_lse, kp_ref, vp_ref = orc.forward_kv8(
        b8.q, b8.k_new, b8.v_new, b8.k_pool, b8.v_pool, ks.numpy(), vs.numpy(), b8.block_table,
        b8.cu_seqlens_q, b8.seq_lens_k, scale=b8.scale, causal=True, page_size=b8.page_size,
        layout=b8.layout, rows=rows)
    assert np.array_equal(kp.numpy(), kp_ref) and np.array_equal(vp.numpy(), vp_ref)
    _check_rows(out, lse, ref, ref_lse, rows, vs, b8, vp_ref)


def test_kv8_mixed_workload_full_size_sampled():
    b8, ks, vs = wl.with_kv8_pools(wl.mixed(), seed=4321)
    out, lse, kp, vp, plan = run_kv8(b8, ks, vs, plan_opts=dict(kv_e4m3=True))
    info = plan.info()
    assert info.num_prefill_tiles > 0 and info.num_decode_items > 0
    rows = _sample_rows(b8, 48, seed=6)
    ref, ref_lse, kp_ref, vp_ref = orc.forward_kv8(
        b8.q, b8.k_new, b8.v_new, b8.k_pool, b8.v_pool, ks.numpy(), vs.numpy(), b8.block_table,
        b8.cu_seqlens_q, b8.seq_lens_k, scale=b8.scale, causal=True, page_size=b8.page_size,
        layout=b8.layout, rows=rows)
    assert np.array_equal(kp.numpy(), kp_ref) and np.array_equal(vp.numpy(), vp_ref)
    _check_rows(out, lse, ref, ref_lse, rows, vs, b8, vp_ref)


@pytest.mark.parametrize("layout", [wl.SEQ_MAJOR, wl.HEAD_MAJOR])
def test_kv8_standalone_write_bit_exact(layout):
    b = wl.ragged_batch([70, 300, 9], [70, 5, 9], 16, 4, 128, 32, seed=980)
    if layout == wl.HEAD_MAJOR:
        b = wl.to_head_major(b)
    b8, ks, vs = wl.with_kv8_pools(b, seed=981)
    plan = plan_for(b8)
    d = {k: getattr(b8, k).cuda().contiguous() for k in (
        "k_new", "v_new", "k_pool", "v_pool", "block_table", "cu_seqlens_q", "seq_lens_k")}
    api.rpa_write_kv8(plan, d["k_new"], d["v_new"], d["k_pool"], d["v_pool"], ks.cuda(),
                      vs.cuda(), d["block_table"], d["cu_seqlens_q"], d["seq_lens_k"])
    torch.cuda.synchronize()
    assert api.rpa_device_error(clear=True) == 0
    kp, vp = orc.write_kv8(b8.k_pool, b8.v_pool, b8.k_new, b8.v_new, ks.numpy(), vs.numpy(),
                           b8.block_table, b8.cu_seqlens_q, b8.seq_lens_k, 32, layout)
    assert np.array_equal(d["k_pool"].cpu().numpy(), kp)
    assert np.array_equal(d["v_pool"].cpu().numpy(), vp)


# ------------------------------------------------------------------ tensor-core kernel on codes

@pytest.mark.parametrize("Hq,Hkv", [(16, 4), (12, 4), (40, 8)])
@pytest.mark.parametrize("layout", [wl.SEQ_MAJOR, wl.HEAD_MAJOR])
def test_kv8_tensor_core_every_code_and_group_size(Hq, Hkv, layout):
    # every finite code (zeros and subnormals included) through the in-kernel expansion;
    # group sizes 4 (query-head pairs), 3 and 5 (one head per unit); NaN codes in every slot
    # past the context: V rows past the last key are zeroed, K columns masked
    b = wl.ragged_batch([700, 260, 129], [400, 260, 129], Hq, Hkv, 128, 32,
                        seed=1000 + Hq + layout, layout=layout)
    b8, ks, vs = wl.with_kv8_pools(b, seed=1001 + Hq, full_range=True)
    out, lse, kp, vp, plan = run_kv8(b8, ks, vs, plan_opts=dict(kv_e4m3=True))
    assert plan.info().num_decode_items == 0 and plan.info().num_prefill_tiles > 0
    ref, ref_lse, kp_ref, vp_ref = oracle_kv8(b8, ks, vs)
    assert np.array_equal(kp.numpy(), kp_ref) and np.array_equal(vp.numpy(), vp_ref)
    check_out(out, ref, vs, b8, vp_ref)
    assert_lse_close(lse, ref_lse)


@pytest.mark.parametrize("scale", [0.3, 4.0])
def test_kv8_tensor_core_large_scores_move_the_reference_max(scale):
    # P is f16 on the e4m3 path: a tile is redone once its row sum passes 2^15, so large
    # score scales (later tiles far above the first tile's max) exercise the redo and the
    # O rescale; the output must stay finite and within the bound
    b = wl.ragged_batch([1500, 700], [900, 700], 8, 2, 128, 64, seed=1010)
    b8, ks, vs = wl.with_kv8_pools(b, seed=1011)
    out, lse, _, _, _ = run_kv8(b8, ks, vs, plan_opts=dict(kv_e4m3=True), scale=scale)
    assert torch.isfinite(out.float()).all()
    ref, ref_lse, _, vp_ref = oracle_kv8(b8, ks, vs, scale=scale)
    check_out(out, ref, vs, b8, vp_ref)
    assert_lse_close(lse, ref_lse)


@pytest.mark.parametrize("page", [16, 64])
def test_kv8_group_tables(page):
    # sparse chunked prefill (block-union group tables) over e4m3 pools
    b = wl.ragged_batch([1500], [300], 8, 2, 128, page, seed=1020 + page, layout=wl.HEAD_MAJOR)
    b8, ks, vs = wl.with_kv8_pools(b, seed=1021)
    mask = wl.structured_block_mask(1, 8, 2, -(-300 // page), b8.max_blocks, seed=1022,
                                    past_blocks=1200 // page)
    table, count = orc.build_group_tables(mask, 2)
    table, count = torch.from_numpy(table), torch.from_numpy(count)
    out, lse, kp, vp, plan = run_kv8(b8, ks, vs, plan_opts=dict(kv_e4m3=True, sparse=True),
                                     group_table=table, group_count=count)
    ref, ref_lse, kp_ref, vp_ref = oracle_kv8(b8, ks, vs, group_table=table.numpy(),
                                              group_count=count.numpy())
    assert np.array_equal(kp.numpy(), kp_ref) and np.array_equal(vp.numpy(), vp_ref)
    check_out(out, ref, vs, b8, vp_ref)
    assert_lse_close(lse, ref_lse)


def test_kv8_query_tile_tables():
    # per-(query tile, head) tables (one head per unit) over e4m3 pools
    b = wl.ragged_batch([1400], [300], 8, 2, 128, 16, seed=1030, layout=wl.HEAD_MAJOR)
    b8, ks, vs = wl.with_kv8_pools(b, seed=1031)
    mask = wl.iid_block_mask(1, 8, -(-300 // 64), b8.max_blocks, seed=1032, density=0.3)
    table, count = orc.build_qtile_tables(mask.numpy(), 64)
    table, count = torch.from_numpy(table), torch.from_numpy(count)
    out, lse, _, _, plan = run_kv8(b8, ks, vs, plan_opts=dict(kv_e4m3=True, sparse=2),
                                   group_table=table, group_count=count)
    ref, ref_lse, _, vp_ref = oracle_kv8(b8, ks, vs, qtile_table=table.numpy(),
                                         qtile_count=count.numpy())
    check_out(out, ref, vs, b8, vp_ref)
    assert_lse_close(lse, ref_lse)


def test_kv8_prefill_workload_full_size_whole_units():
    # the prefill workload (4 x 4096 causal, page 64) over e4m3 pools, persistent grid as for
    # bf16: whole units (128 rows x both heads of a pair) of the first, a middle and the last
    # tile of every sequence, and units of the walk's first and second rounds
    b8, ks, vs = wl.with_kv8_pools(wl.prefill(), seed=1040)
    out, lse, kp, vp, plan = run_kv8(b8, ks, vs, plan_opts=dict(kv_e4m3=True))
    assert plan.info().num_prefill_tiles == 128
    cu = b8.cu_seqlens_q.tolist()
    units = [(s, t, h) for s in range(4) for t, h in ((0, 0), (15, 14), (31, 30))]
    units += [(0, 31, 0), (1, 30, 10), (1, 29, 16), (0, 28, 6)]
    rows = sorted({(cu[s] + i, h + x) for s, t, h in units for i in range(t * 128, t * 128 + 128)
                   for x in (0, 1)})
    ref, ref_lse, kp_ref, vp_ref = oracle_kv8(b8, ks, vs, rows=rows)
    assert np.array_equal(kp.numpy(), kp_ref) and np.array_equal(vp.numpy(), vp_ref)
    check_out(out, ref, vs, b8, vp_ref, rows=rows)
    for t, h in rows[::97]:
        assert abs(float(lse[t, h]) - ref_lse[t, h]) <= 2e-3, (t, h)
