"""GPU parity of the block-sparse execution (per-(query tile, query head) tables, one head
per CTA) used by the execution-only ablation: the table builder bit for bit, attention
against the oracle, and identity with the per-group-table execution on the unioned mask."""
import numpy as np
import pytest
import torch

from oracle import rpa_oracle as orc
from ragged_paged_attention_forward_b200 import api
from ragged_paged_attention_forward_b200 import workloads as wl
from tests.rpa_testing import assert_close, assert_lse_close, run_forward

pytestmark = pytest.mark.gpu


def _gpu_qtile_tables(mask, q_block_rows):
    B, Hq, nqb, nkb = mask.shape
    nt = -(-nqb // (128 // q_block_rows))
    table = torch.full((B, Hq, nt, nkb), 7, dtype=torch.int32, device="cuda")
    count = torch.full((B, Hq, nt), 7, dtype=torch.int32, device="cuda")
    api.rpa_build_qtile_tables(torch.from_numpy(mask).cuda(), q_block_rows, table, count)
    torch.cuda.synchronize()
    return table, count


@pytest.mark.parametrize("qbr", [32, 64, 128])
def test_qtile_tables_bit_exact(qbr):
    rng = np.random.default_rng(500 + qbr)
    mask = (rng.random((2, 8, 9, 300)) < 0.1).astype(np.uint8)
    table, count = _gpu_qtile_tables(mask, qbr)
    rt, rc = orc.build_qtile_tables(mask, qbr)
    assert np.array_equal(table.cpu().numpy(), rt) and np.array_equal(count.cpu().numpy(), rc)


def _case(kv_len, chunk, page, seed, Hq=8, Hkv=2):
    b = wl.ragged_batch([kv_len], [chunk], Hq, Hkv, 128, page, seed=seed, layout=wl.HEAD_MAJOR)
    nqb = -(-chunk // 64)
    mask = wl.iid_block_mask(1, Hq, nqb, b.max_blocks, seed=seed + 1, density=0.3)
    return b, mask


def _oracle_qtile(b, table, count):
    return orc.forward(b.q, b.k_new, b.v_new, b.k_pool, b.v_pool, b.block_table,
                       b.cu_seqlens_q, b.seq_lens_k, scale=b.scale, causal=b.causal,
                       page_size=b.page_size, layout=b.layout, qtile_table=table,
                       qtile_count=count)


@pytest.mark.parametrize("page", [16, 64])
def test_qtile_forward_matches_oracle(page):
    b, mask = _case(1400, 300, page, seed=510 + page)
    table, count = _gpu_qtile_tables(mask.numpy() if hasattr(mask, "numpy") else mask, 64)
    out, lse, _, _, plan = run_forward(b, group_table=table, group_count=count,
                                       plan_opts=dict(sparse=2))
    assert plan.info().num_decode_items == 0
    ref, ref_lse, _, _ = _oracle_qtile(b, table.cpu().numpy(), count.cpu().numpy())
    assert_close(out, ref)
    assert_lse_close(lse, ref_lse)


def test_qtile_on_the_unioned_mask_equals_group_tables_bit_for_bit():
    b, mask = _case(2000, 384, 64, seed=520)
    m = mask.numpy() if hasattr(mask, "numpy") else mask
    gt, gc = orc.build_group_tables(m, 2)
    out_g, lse_g, _, _, _ = run_forward(b, group_table=torch.from_numpy(gt),
                                        group_count=torch.from_numpy(gc))
    B, Hq, nqb, nkb = m.shape
    u = np.zeros_like(m)
    for g in range(2):
        u[0, g * 4:(g + 1) * 4, :, gt[0, g, :gc[0, g]]] = 1
    table, count = _gpu_qtile_tables(u, 64)
    out_q, lse_q, _, _, _ = run_forward(b, group_table=table, group_count=count,
                                        plan_opts=dict(sparse=2))
    # the same tiles, keys and arithmetic per row: one head per CTA changes no row's result
    assert torch.equal(out_g.view(torch.int16), out_q.view(torch.int16))
    assert torch.equal(lse_g, lse_q)


def test_qtile_sparse_workload_full_size_sampled():
    # the benchmark's sparse configuration (2048 queries at 128K context) run block-sparse per
    # (query tile, head) on the original per-head mask; sampled rows against the oracle
    b, mask = wl.sparse()
    m = mask.numpy()
    table, count = _gpu_qtile_tables(m, b.num_tokens // m.shape[2])
    out, lse, _, _, _ = run_forward(b, group_table=table, group_count=count,
                                    plan_opts=dict(sparse=2))
    g = np.random.default_rng(7)
    rows = sorted({(int(t), int(h)) for t, h in zip(g.integers(0, b.num_tokens, 24),
                                                    g.integers(0, b.num_q_heads, 24))})
    ref, ref_lse, _, _ = orc.forward(b.q, b.k_new, b.v_new, b.k_pool, b.v_pool, b.block_table,
                                     b.cu_seqlens_q, b.seq_lens_k, scale=b.scale, causal=True,
                                     page_size=b.page_size, layout=b.layout,
                                     qtile_table=table.cpu().numpy(),
                                     qtile_count=count.cpu().numpy(), rows=rows)
    assert_close(out, ref, rows=rows)
    assert_lse_close(lse, ref_lse, rows=rows)
