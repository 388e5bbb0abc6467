"""GPU parity of the e4m3 (fp8) KV-cache decode path against the fp64 oracle.

The quantising KV write must produce the oracle's codes bit for bit; attention over the
dequantised cache must match within the tolerance derived below.  Runs through the C ABI
(rpa_forward_kv8)."""
import numpy as np
import pytest
import torch

from oracle import rpa_oracle as orc
from ragged_paged_attention_forward_b200 import api
from ragged_paged_attention_forward_b200 import workloads as wl
from tests.rpa_testing import assert_kv8_close, assert_lse_close, kv8_vmax, plan_for

pytestmark = pytest.mark.gpu


def run_kv8(b8, ks, vs, *, plan_opts=None, with_new=True):
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
                        d["seq_lens_k"], b8.scale, out, lse, ws)
    torch.cuda.synchronize()
    assert api.rpa_device_error(clear=True) == 0
    return out.cpu(), lse.cpu(), d["k_pool"].cpu(), d["v_pool"].cpu(), plan


def oracle_kv8(b8, ks, vs, with_new=True):
    return orc.forward_kv8(b8.q, b8.k_new if with_new else None, b8.v_new if with_new else None,
                           b8.k_pool, b8.v_pool, ks.numpy(), vs.numpy(), b8.block_table,
                           b8.cu_seqlens_q, b8.seq_lens_k, scale=b8.scale, causal=b8.causal,
                           page_size=b8.page_size, layout=b8.layout)


def check_out(out, ref, vs, b8, v_pool_after, rows=None):
    # the bound of tests.rpa_testing.kv8_output_errors (derived there): pointwise
    # 2^-8 (max|V| + |o|) with max|V| what the written V pool holds, and mean-abs <= 2e-3
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
    # decode rows on the e4m3 pools directly; prefill chunks (with past) on the exact bf16
    # copy of their context; the new tokens of both quantised by the scatter kernel
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
