"""GPU parity of the KV write, the split-KV decode path (short query rows) and the group-table
builder against the fp64 oracle, through the C ABI."""
import math

import numpy as np
import pytest
import torch

from oracle import rpa_oracle as orc
from ragged_paged_attention_forward_b200 import api
from ragged_paged_attention_forward_b200 import workloads as wl
from tests.rpa_testing import (assert_close, assert_lse_close, oracle_forward, run_forward,
                               to_device, plan_for)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("layout", [wl.SEQ_MAJOR, wl.HEAD_MAJOR])
@pytest.mark.parametrize("page", [16, 64, 256])
def test_write_kv_bit_exact_whole_pool(layout, page):
    b = wl.ragged_batch([1, 17, 300, 64, 129], [1, 17, 37, 3, 2], 8, 2, 128, page, seed=31,
                        layout=layout)
    plan = plan_for(b)
    d = to_device(b)
    api.rpa_write_kv(plan, d["k_new"], d["v_new"], d["k_pool"], d["v_pool"], d["block_table"],
                     d["cu_seqlens_q"], d["seq_lens_k"])
    torch.cuda.synchronize()
    assert api.rpa_device_error() == 0
    kp, vp = orc.write_kv(b.k_pool, b.v_pool, b.k_new, b.v_new, b.block_table, b.cu_seqlens_q,
                          b.seq_lens_k, b.page_size, b.layout)
    assert np.array_equal(orc.bits16(d["k_pool"].cpu()), kp)
    assert np.array_equal(orc.bits16(d["v_pool"].cpu()), vp)


def test_tiny_config_fused_and_split_write():
    b = wl.tiny()
    ref, ref_lse, kp, vp = oracle_forward(b)
    for fused in (True, False):
        out, lse, gk, gv, _ = run_forward(b, fused=fused)
        assert_close(out, ref)
        assert_lse_close(lse, ref_lse)
        assert np.array_equal(orc.bits16(gk), kp) and np.array_equal(orc.bits16(gv), vp)


def test_decode_config_full_size():
    b = wl.decode()
    out, lse, gk, gv, plan = run_forward(b)
    assert plan.info().batch_class == api.CLASS_DECODE
    ref, ref_lse, kp, vp = oracle_forward(b)
    assert_close(out, ref)
    assert_lse_close(lse, ref_lse)
    assert np.array_equal(orc.bits16(gk), kp)


@pytest.mark.parametrize("split", [64, 256, 1024, 4096])
def test_decode_split_sizes_agree(split):
    b = wl.ragged_batch([50, 700, 2500, 4100, 65], [1, 1, 1, 1, 1], 32, 8, 128, 16, seed=32)
    ref, ref_lse, _, _ = oracle_forward(b)
    out, lse, _, _, plan = run_forward(b, plan_opts=dict(decode_split_keys=split))
    assert plan.info().decode_split_keys == split
    assert_close(out, ref)
    assert_lse_close(lse, ref_lse)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (32, 8), (16, 2), (32, 1)])
@pytest.mark.parametrize("page", [16, 32, 128])
def test_decode_grid(D, Hq, Hkv, page):
    kv = [1, 15, 16, 17, 64, 100, 333, 1024]
    b = wl.ragged_batch(kv, [1] * len(kv), Hq, Hkv, D, page, seed=33 + D + Hq + page)
    ref, ref_lse, _, _ = oracle_forward(b)
    out, lse, _, _, plan = run_forward(b, plan_opts=dict(decode_split_keys=256))
    assert plan.info().num_decode_items > 0
    assert_close(out, ref)
    assert_lse_close(lse, ref_lse)


@pytest.mark.parametrize("causal", [True, False])
def test_short_multi_token_rows_on_decode_kernel(causal):
    # q_len * G <= 16 goes to the decode kernel in a mixed batch; q_len 2..4 with past > 0
    b = wl.ragged_batch([40, 300, 77, 1000], [2, 4, 3, 1], 8, 2, 128, 16, seed=34,
                        causal=causal)
    ref, ref_lse, _, _ = oracle_forward(b)
    out, lse, _, _, plan = run_forward(b, plan_opts=dict(decode_split_keys=128))
    info = plan.info()
    assert info.num_prefill_tiles == 0 and info.num_decode_items > 0
    assert_close(out, ref)
    assert_lse_close(lse, ref_lse)


def test_decode_head_major_layout_and_scale():
    b = wl.to_head_major(wl.ragged_batch([90, 513, 2049], [1, 1, 1], 32, 8, 128, 16, seed=35))
    ref, ref_lse, _, _ = oracle_forward(b, scale=0.05)
    out, lse, _, _, _ = run_forward(b, scale=0.05, plan_opts=dict(decode_split_keys=512))
    assert_close(out, ref)
    assert_lse_close(lse, ref_lse)


def test_decode_page_permutation_gives_identical_output():
    b = wl.ragged_batch([700, 1500, 33], [1, 1, 1], 32, 8, 128, 16, seed=36)
    b2 = wl.permute_pages(b, seed=7)
    o1 = run_forward(b)[0]
    o2 = run_forward(b2)[0]
    assert torch.equal(o1, o2)


def test_empty_sequences_and_zero_tokens():
    b = wl.ragged_batch([30, 50, 70], [1, 0, 1], 8, 2, 64, 16, seed=37)
    ref, _, _, _ = oracle_forward(b)
    out, _, _, _, _ = run_forward(b)
    assert_close(out, ref)
    z = wl.ragged_batch([30, 50], [0, 0], 8, 2, 64, 16, seed=38)
    out, _, gk, _, plan = run_forward(z)
    assert out.numel() == 0
    assert torch.equal(gk, z.k_pool) or torch.equal(gk.isnan(), z.k_pool.isnan())


def _tables_on_gpu(mask, Hkv):
    B, Hq, nqb, nkb = mask.shape
    m = mask.cuda()
    table = torch.full((B, Hkv, nkb), 12345, dtype=torch.int32, device="cuda")
    count = torch.full((B, Hkv), -7, dtype=torch.int32, device="cuda")
    api.rpa_build_group_tables(m, Hkv, table, count)
    torch.cuda.synchronize()
    return table.cpu().numpy(), count.cpu().numpy()


@pytest.mark.parametrize("density", [0.0, 0.01, 0.3, 1.0])
def test_group_tables_bit_exact_iid(density):
    mask = wl.iid_block_mask(3, 8, 5, 1300, seed=40, density=density)
    t, c = _tables_on_gpu(mask, 2)
    rt, rc = orc.build_group_tables(mask, 2)
    assert np.array_equal(t, rt) and np.array_equal(c, rc)


def test_group_tables_bit_exact_sparse_config_mask():
    mask = wl.sparse_mask()
    t, c = _tables_on_gpu(mask, 8)
    rt, rc = orc.build_group_tables(mask, 8)
    assert np.array_equal(t, rt) and np.array_equal(c, rc)
    density = rc.sum() / (8 * mask.shape[-1])
    assert 0.15 < density < 0.35


@pytest.mark.parametrize("nkb,nqb,density", [(16, 1, 0.5), (2048, 32, 0.02), (4128, 3, 0.3),
                                              (4096, 2, 0.0), (64, 5, 1.0)])
def test_group_tables_bit_exact_vector_path(nkb, nqb, density):
    mask = wl.iid_block_mask(2, 8, nqb, nkb, seed=41 + nkb, density=density)
    t, c = _tables_on_gpu(mask, 4)
    rt, rc = orc.build_group_tables(mask, 4)
    assert np.array_equal(t, rt) and np.array_equal(c, rc)


def test_bounded_wait_runs_out_reports_and_leaves_the_context_usable():
    # Failure detection without a GPU fault: with the diagnostic plan option the decode
    # kernel issues no K/V copy, so its consumers' waits on the copies can only run out.  They
    # give up after 2 ms (not the normal 2 s), record bit 1 in the device error word and the
    # kernel returns; nothing is left in flight.  The next normal step on the same context
    # must be correct.
    import time
    b = wl.ragged_batch([300, 1025, 64], [1, 1, 1], 32, 8, 128, 16, seed=111)
    assert api.rpa_device_error(clear=True) == 0
    plan = plan_for(b, wait_test_us=2000)
    assert plan.info().batch_class == api.CLASS_DECODE
    d = to_device(b)
    out = torch.zeros_like(d["q"])
    ws = torch.empty(max(plan.workspace_bytes, 256), dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    api.rpa_forward(plan, d["q"], d["k_new"], d["v_new"], d["k_pool"], d["v_pool"],
                    d["block_table"], d["cu_seqlens_q"], d["seq_lens_k"], None, None, b.scale,
                    out, None, ws)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert api.rpa_device_error(clear=True) == 1     # decode wait ran out, nothing else
    assert elapsed < 1.0, elapsed                     # well before the normal 2 s limit
    ref, ref_lse, kp, vp = oracle_forward(b)
    out, lse, gk, gv, _ = run_forward(b)
    assert_close(out, ref)
    assert_lse_close(lse, ref_lse)
    assert np.array_equal(orc.bits16(gk), kp) and np.array_equal(orc.bits16(gv), vp)
