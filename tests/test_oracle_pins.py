"""Pins for the fp64 oracle: each test checks it against something other than itself --
hand-derived fixtures, a library routine (torch SDPA / logsumexp), closed forms, invariants
and brute force -- chosen so that a dropped term, a wrong sign or index, or a transposed
operand in the oracle fails at least one of them.  CPU only."""
import itertools
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import rpa_oracle as orc
from ragged_paged_attention_forward_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _oracle_forward(batch, **kw):
    return orc.forward(batch.q, batch.k_new, batch.v_new, batch.k_pool, batch.v_pool,
                       batch.block_table, batch.cu_seqlens_q, batch.seq_lens_k,
                       scale=kw.pop("scale", batch.scale), causal=kw.pop("causal", batch.causal),
                       page_size=batch.page_size, layout=batch.layout, **kw)


def _f64(t):
    return t.to(torch.float64)


def _sdpa_row(q_row, K, V, scale):
    """Library attention (torch SDPA, fp64, no mask) of one query row over rows K, V."""
    o = F.scaled_dot_product_attention(q_row.view(1, 1, -1), K.unsqueeze(0), V.unsqueeze(0),
                                       scale=scale)
    return o.view(-1).numpy()


# ------------------------------------------------------------------------------------
# KV write
# ------------------------------------------------------------------------------------

def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def test_scatter_matches_hand_derived_slots():
    P, Hkv, D = 16, 2, 8
    kv_lens, q_lens = [19, 33], [2, 3]
    bt = np.array([[5, 2, 9], [7, 0, 4]], dtype=np.int32)
    cu = np.array([0, 2, 5], dtype=np.int32)
    sentinel = np.uint16(0x7FC1)
    kp = np.full((10, P, Hkv, D), sentinel, dtype=np.uint16)
    vp = np.full((10, P, Hkv, D), sentinel, dtype=np.uint16)
    T = 5
    kn = (np.arange(T * Hkv * D, dtype=np.uint16).reshape(T, Hkv, D) + 0x3F00)
    vn = (np.arange(T * Hkv * D, dtype=np.uint16).reshape(T, Hkv, D) + 0x4000)
    kp2, vp2 = orc.write_kv(kp, vp, kn, vn, bt, cu, np.array(kv_lens, dtype=np.int32), P)
    expected = {}
    for tok, page, slot in _read_golden("scatter_tiny.txt"):
        expected[(int(page), int(slot))] = int(tok)
    for page in range(10):
        for slot in range(P):
            if (page, slot) in expected:
                t = expected[(page, slot)]
                assert np.array_equal(kp2[page, slot], kn[t])
                assert np.array_equal(vp2[page, slot], vn[t])
            else:
                assert np.all(kp2[page, slot] == sentinel)
                assert np.all(vp2[page, slot] == sentinel)


@pytest.mark.parametrize("layout", [wl.SEQ_MAJOR, wl.HEAD_MAJOR])
def test_write_then_gather_returns_logical_sequence(layout):
    b = wl.ragged_batch([1, 17, 40, 64, 65], [1, 5, 40, 3, 2], 4, 2, 16, 16, seed=11,
                        layout=layout)
    kp, vp = orc.write_kv(b.k_pool, b.v_pool, b.k_new, b.v_new, b.block_table,
                          b.cu_seqlens_q, b.seq_lens_k, b.page_size, b.layout)
    for s, kv in enumerate(b.kv_lens()):
        for h in range(b.num_kv_heads):
            got_k = orc.logical_rows(kp, b.block_table, layout, s, h, kv, b.page_size)
            got_v = orc.logical_rows(vp, b.block_table, layout, s, h, kv, b.page_size)
            assert np.array_equal(got_k, orc.bits16(b.k_logical[s][:, h]))
            assert np.array_equal(got_v, orc.bits16(b.v_logical[s][:, h]))
    # bytes the write must not touch keep their poison pattern
    before = orc.bits16(b.k_pool)
    changed = np.any(kp != before, axis=tuple(range(1, kp.ndim)))
    assert int(changed.sum()) <= sum(math.ceil(q / b.page_size) + 1 for q in b.q_lens()) * (
        b.num_kv_heads if layout == wl.HEAD_MAJOR else 1)


# ------------------------------------------------------------------------------------
# Attention against a library routine and against closed forms
# ------------------------------------------------------------------------------------

def _sdpa_reference(batch, scale=None):
    """Attention of each row as torch SDPA over the *logical* (unpaged) prefix of keys the
    row may see; uses the generator's logical rows, never the pool."""
    scale = batch.scale if scale is None else scale
    G = batch.num_q_heads // batch.num_kv_heads
    T, Hq, D = batch.q.shape
    out = np.zeros((T, Hq, D))
    cu = batch.cu_seqlens_q.tolist()
    for s, kv in enumerate(batch.kv_lens()):
        q_len = cu[s + 1] - cu[s]
        past = kv - q_len
        for i in range(q_len):
            t = cu[s] + i
            n = min(kv, past + i + 1) if batch.causal else kv
            for hq in range(Hq):
                K = _f64(batch.k_logical[s][:n, hq // G])
                V = _f64(batch.v_logical[s][:n, hq // G])
                out[t, hq] = _sdpa_row(_f64(batch.q[t, hq]), K, V, scale)
    return out


@pytest.mark.parametrize("case", ["tiny", "ragged", "mha", "noncausal"])
def test_oracle_equals_library_attention_over_logical_prefix(case):
    if case == "tiny":
        b = wl.tiny()
    elif case == "ragged":
        b = wl.ragged_batch([5, 70, 33, 129], [5, 1, 17, 40], 8, 2, 32, 16, seed=3)
    elif case == "mha":
        b = wl.ragged_batch([9, 48], [3, 48], 3, 3, 16, 32, seed=4, scale=0.37)
    else:
        b = wl.ragged_batch([20, 35], [4, 6], 4, 1, 16, 16, seed=5, causal=False)
    out, lse, _, _ = _oracle_forward(b)
    ref = _sdpa_reference(b)
    assert np.max(np.abs(out - ref)) < 1e-12


def test_causal_prefill_without_past_equals_library_causal_mask():
    b = wl.ragged_batch([37], [37], 2, 2, 16, 16, seed=6)
    out, _, _, _ = _oracle_forward(b)
    q = _f64(b.q).permute(1, 0, 2)                     # [H, T, D]
    k = _f64(b.k_logical[0]).permute(1, 0, 2)
    v = _f64(b.v_logical[0]).permute(1, 0, 2)
    ref = F.scaled_dot_product_attention(q, k, v, is_causal=True, scale=b.scale)
    assert np.max(np.abs(out - ref.permute(1, 0, 2).numpy())) < 1e-12


def test_causal_boundary_by_perturbation():
    """Row at absolute position p must change when key/value p changes and must not change
    when any key/value after p changes (mixed q_len with past > 0)."""
    b = wl.ragged_batch([30, 12], [6, 12], 2, 1, 16, 16, seed=8)
    out, _, kp, vp = _oracle_forward(b)
    seqs = orc.seq_ranges(b.cu_seqlens_q, b.seq_lens_k)
    for s, (t0, q_len, kv_len, past) in enumerate(seqs):
        for i in range(q_len):
            p = past + i
            for j, expect_change in ((p, True), (p + 1, False), (kv_len - 1, p == kv_len - 1)):
                if j >= kv_len:
                    continue
                kp2, vp2 = kp.copy(), vp.copy()
                page = int(b.block_table[s, j // b.page_size])
                vp2[page, j % b.page_size] = orc.bits16(
                    torch.full((b.num_kv_heads, b.head_dim), 3.0, dtype=torch.bfloat16))
                o2, _ = orc.attention(b.q, kp2, vp2, b.block_table, b.cu_seqlens_q,
                                      b.seq_lens_k, scale=b.scale, causal=True,
                                      page_size=b.page_size, num_kv_heads=b.num_kv_heads,
                                      rows=[(t0 + i, 0)])
                changed = not np.array_equal(o2[t0 + i, 0], out[t0 + i, 0])
                assert changed == expect_change, (s, i, j)


def test_constant_values_return_that_value():
    b = wl.ragged_batch([3, 50, 130], [3, 1, 9], 4, 2, 16, 16, seed=9)
    c = torch.randn(2, 16, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    b.v_new[:] = c
    vp = b.v_pool.clone()
    used = ~torch.isnan(vp.float())
    vp[used] = c.unsqueeze(0).unsqueeze(0).expand_as(vp)[used]
    b.v_pool = vp
    out, _, _, _ = _oracle_forward(b)
    G = 2
    expect = _f64(c)[torch.arange(4) // G].numpy()
    for t in range(b.num_tokens):
        assert np.max(np.abs(out[t] - expect)) <= 4e-16 * np.max(np.abs(expect)) * 10


def test_single_visible_key_gets_weight_one():
    # kv_len 1 decode, and row 0 of a prefill without past
    b = wl.ragged_batch([1, 7], [1, 7], 2, 2, 16, 16, seed=10)
    out, lse, _, _ = _oracle_forward(b)
    for t, s in ((0, 0), (1, 1)):
        for hq in range(2):
            v0 = orc.widen(orc.bits16(b.v_logical[s][0, hq]))
            k0 = orc.widen(orc.bits16(b.k_logical[s][0, hq]))
            assert np.array_equal(out[t, hq], v0)
            q = orc.widen(orc.bits16(b.q[t, hq]))
            assert lse[t, hq] == pytest.approx(b.scale * float(q @ k0), abs=1e-14)


def test_zero_scale_gives_mean_and_log_count():
    b = wl.ragged_batch([10, 64], [4, 2], 2, 1, 16, 16, seed=12)
    out, lse, _, _ = _oracle_forward(b, scale=0.0)
    seqs = orc.seq_ranges(b.cu_seqlens_q, b.seq_lens_k)
    for s, (t0, q_len, kv_len, past) in enumerate(seqs):
        for i in range(q_len):
            n = past + i + 1
            mean = _f64(b.v_logical[s][:n, 0]).mean(0).numpy()
            for hq in range(2):
                assert np.max(np.abs(out[t0 + i, hq] - mean)) < 1e-14
                assert lse[t0 + i, hq] == pytest.approx(math.log(n), abs=1e-14)


def test_one_dominant_key_closed_form():
    """All keys zero except key m = a*e_0: o = (e^s v_m + sum_{j!=m} v_j) / (e^s + n - 1)
    with s = scale * a * q_0."""
    b = wl.ragged_batch([40], [1], 1, 1, 16, 16, seed=13, causal=False)
    m, a = 17, 4.0
    kp = torch.zeros_like(b.k_pool)
    page = int(b.block_table[0, m // 16])
    kp[page, m % 16, 0, 0] = a
    b.k_pool = kp
    b.k_new = torch.zeros_like(b.k_new)
    out, lse, _, vp = _oracle_forward(b)
    q0 = float(_f64(b.q[0, 0, 0]))
    s = b.scale * a * q0
    V = orc.widen(orc.logical_rows(vp, b.block_table, 0, 0, 0, 40, 16))
    expect = (math.exp(s) * V[m] + V.sum(0) - V[m]) / (math.exp(s) + 39)
    assert np.max(np.abs(out[0, 0] - expect)) < 1e-13
    assert lse[0, 0] == pytest.approx(math.log(math.exp(s) + 39), abs=1e-13)


def test_lse_matches_library_logsumexp():
    b = wl.ragged_batch([33, 8], [5, 8], 4, 2, 16, 16, seed=14)
    _, lse, kp, _ = _oracle_forward(b)
    seqs = orc.seq_ranges(b.cu_seqlens_q, b.seq_lens_k)
    for s, (t0, q_len, kv_len, past) in enumerate(seqs):
        for i in range(q_len):
            for hq in range(4):
                K = _f64(b.k_logical[s][:past + i + 1, hq // 2])
                ref = torch.logsumexp(b.scale * (K @ _f64(b.q[t0 + i, hq])), 0).item()
                assert lse[t0 + i, hq] == pytest.approx(ref, abs=1e-12)


def test_gqa_equals_mha_with_replicated_kv_heads():
    b = wl.ragged_batch([21, 50], [3, 50], 8, 2, 16, 16, seed=15)
    G = 4
    mha = wl.ragged_batch([21, 50], [3, 50], 8, 8, 16, 16, seed=15)
    mha.q = b.q
    mha.k_new = b.k_new.repeat_interleave(G, dim=1)
    mha.v_new = b.v_new.repeat_interleave(G, dim=1)
    mha.block_table = b.block_table
    mha.k_pool = b.k_pool.repeat_interleave(G, dim=2)
    mha.v_pool = b.v_pool.repeat_interleave(G, dim=2)
    o1, l1, _, _ = _oracle_forward(b)
    o2, l2, _, _ = _oracle_forward(mha)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_page_permutation_invariance_is_bit_exact():
    b = wl.ragged_batch([17, 64, 130, 5], [1, 1, 5, 5], 4, 2, 32, 16, seed=16)
    b2 = wl.permute_pages(b, seed=99)
    assert not torch.equal(b.block_table, b2.block_table)
    o1, l1, _, _ = _oracle_forward(b)
    o2, l2, _, _ = _oracle_forward(b2)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_head_major_equals_seq_major_bit_exact():
    b = wl.ragged_batch([17, 64, 130], [1, 30, 5], 4, 2, 32, 16, seed=17)
    hm = wl.to_head_major(b)
    o1, l1, kp, _ = _oracle_forward(b)
    o2, l2, kph, _ = _oracle_forward(hm)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_split_merge_equals_unsplit():
    g = np.random.default_rng(0)
    b = wl.ragged_batch([300], [1], 1, 1, 64, 16, seed=18)
    _, _, kp, vp = _oracle_forward(b)
    K = orc.widen(orc.logical_rows(kp, b.block_table, 0, 0, 0, 300, 16))
    V = orc.widen(orc.logical_rows(vp, b.block_table, 0, 0, 0, 300, 16))
    q = orc.widen(orc.bits16(b.q[0, 0]))
    whole = orc.attend_row(q, K, V, b.scale)
    for cuts in ([150], [16, 64, 200], sorted(g.choice(np.arange(1, 300), 9, replace=False))):
        edges = [0] + list(cuts) + [300]
        parts = [orc.attend_row(q, K[a:c], V[a:c], b.scale) for a, c in zip(edges, edges[1:])]
        parts.append(orc.attend_row(q, K[:0], V[:0], b.scale))   # an empty split
        o, l = orc.merge_partials(parts)
        assert np.max(np.abs(o - whole[0])) < 1e-12
        assert l == pytest.approx(whole[1], abs=1e-12)


# ------------------------------------------------------------------------------------
# Block-union tables
# ------------------------------------------------------------------------------------

def test_group_tables_hand_derived_fixture():
    rows = _read_golden("group_tables_tiny.txt")
    mask = np.zeros((1, 4, 2, 5), dtype=np.uint8)
    expect = {}
    for r in rows:
        if r[0] == "mask":
            mask[0, int(r[1]), int(r[2])] = [int(x) for x in r[3:]]
        else:
            expect[int(r[1])] = (int(r[2]), [int(x) for x in r[3:]])
    table, count = orc.build_group_tables(mask, 2)
    for g, (n, entries) in expect.items():
        assert count[0, g] == n
        assert table[0, g].tolist() == entries


@pytest.mark.parametrize("Hq,Hkv,nqb,nkb", [(4, 2, 2, 2), (2, 1, 2, 3), (4, 1, 1, 4)])
def test_group_tables_exhaustive(Hq, Hkv, nqb, nkb):
    """Every mask of the shape: a block is listed for a group iff some query head of the
    group selects it in some query block (complete and minimal); ascending, no duplicates."""
    G = Hq // Hkv
    nbits = Hq * nqb * nkb
    bits = ((np.arange(2 ** nbits)[:, None] >> np.arange(nbits)) & 1).astype(np.uint8)
    for code in range(2 ** nbits):
        mask = bits[code].reshape(1, Hq, nqb, nkb)
        table, count = orc.build_group_tables(mask, Hkv)
        for g in range(Hkv):
            need = [kb for kb in range(nkb)
                    if any(mask[0, hq, qb, kb] for hq in range(g * G, (g + 1) * G)
                           for qb in range(nqb))]
            n = int(count[0, g])
            assert table[0, g, :n].tolist() == need
            assert all(x == -1 for x in table[0, g, n:])


def test_sparse_all_ones_equals_dense_and_truncation():
    P = 16
    b = wl.ragged_batch([200], [40], 4, 2, 16, P, seed=19, layout=wl.HEAD_MAJOR)
    nkb = math.ceil(200 / P)
    dense, dlse, _, _ = _oracle_forward(b)
    ones = np.ones((1, 4, 3, nkb), dtype=np.uint8)
    table, count = orc.build_group_tables(ones, 2)
    o1, l1, _, _ = _oracle_forward(b, group_table=table, group_count=count)
    assert np.array_equal(o1, dense) and np.array_equal(l1, dlse)
    # keep blocks 0..c only: equals attention over the prefix min(p+1, (c+1)*P)
    c = 7
    trunc = np.zeros_like(ones)
    trunc[..., :c + 1] = 1
    table, count = orc.build_group_tables(trunc, 2)
    o2, _, _, _ = _oracle_forward(b, group_table=table, group_count=count)
    past = 160
    for i in range(40):
        n = min(past + i + 1, (c + 1) * P)
        for hq in range(4):
            K = _f64(b.k_logical[0][:n, hq // 2])
            V = _f64(b.v_logical[0][:n, hq // 2])
            ref = _sdpa_row(_f64(b.q[i, hq]), K, V, b.scale)
            assert np.max(np.abs(o2[i, hq] - ref)) < 1e-12


def test_sparse_row_with_no_visible_block_is_zero():
    P = 16
    b = wl.ragged_batch([64], [64], 2, 1, 16, P, seed=20, layout=wl.HEAD_MAJOR)
    mask = np.zeros((1, 2, 1, 4), dtype=np.uint8)
    mask[..., 3] = 1            # only the last block: rows before position 48 see nothing
    table, count = orc.build_group_tables(mask, 1)
    out, lse, _, _ = _oracle_forward(b, group_table=table, group_count=count)
    assert np.all(out[:48] == 0) and np.all(np.isneginf(lse[:48]))
    assert np.all(np.isfinite(lse[48:]))


def test_tolerance_is_reachable_with_bf16_inputs_and_fp32_accumulation():
    """An fp32-accumulating computation that rounds P to bf16 stays well inside
    max-abs 2e-2 / mean-abs 2e-3 of the fp64 oracle on a decode-shaped batch."""
    b = wl.ragged_batch([700, 1500, 2300], [1, 1, 1], 32, 8, 128, 16, seed=21)
    out, _, _, _ = _oracle_forward(b)
    err = []
    for s, kv in enumerate(b.kv_lens()):
        for hq in range(32):
            K = b.k_logical[s][:, hq // 4].float()
            V = b.v_logical[s][:, hq // 4].float()
            sc = (K @ b.q[s, hq].float()) * b.scale
            p = torch.exp(sc - sc.max())
            o = (p.to(torch.bfloat16).float() @ V) / p.sum()
            err.append(np.abs(o.to(torch.bfloat16).double().numpy() - out[s, hq]))
    err = np.concatenate(err)
    assert err.max() < 2e-2 / 4 and err.mean() < 2e-3 / 4


# ------------------------------------------------------------------------------------
# Rotary position embedding, packed QKV, bf16 rounding (the input pass)
# ------------------------------------------------------------------------------------

def _bf16_bits_from_f32(v):
    return torch.tensor(v, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy() \
        .view(np.uint16)


def test_round_bf16_matches_torch_on_fp32_values_and_ties():
    # fp32-representable values round the same through torch's fp32 -> bf16 conversion
    g = np.random.default_rng(3)
    x = g.standard_normal(4000).astype(np.float32) * np.float32(10.0) ** g.integers(-30, 30, 4000)
    assert np.array_equal(orc.round_bf16(x.astype(np.float64)), _bf16_bits_from_f32(x))
    # exact ties go to the even significand: 1 + 2^-8 -> 1, 1 + 3*2^-8 -> 1 + 2^-6
    assert orc.round_bf16(np.array([1 + 2 ** -8]))[0] == 0x3F80
    assert orc.round_bf16(np.array([1 + 3 * 2 ** -8]))[0] == 0x3F82
    # a value just above a tie rounds up although its fp32 rounding would be the tie itself
    assert orc.round_bf16(np.array([1 + 2 ** -8 + 2 ** -40]))[0] == 0x3F81


def _unit_angles(n, half, seed):
    g = np.random.default_rng(seed)
    theta = g.uniform(-math.pi, math.pi, (n, half))
    return np.cos(theta), np.sin(theta), theta


def test_rotate_split_is_complex_multiplication():
    D, rd = 16, 12
    cos, sin, theta = _unit_angles(5, rd // 2, 1)
    x = np.random.default_rng(2).standard_normal((7, D))
    pos = np.array([0, 4, 2, 2, 3, 1, 0])
    out = orc.rotate(x, pos, cos, sin, rd, interleaved=False)
    z = (x[:, :rd // 2] + 1j * x[:, rd // 2:rd]) * np.exp(1j * theta[pos])
    assert np.allclose(out[:, :rd // 2], z.real, rtol=0, atol=1e-12)
    assert np.allclose(out[:, rd // 2:rd], z.imag, rtol=0, atol=1e-12)
    assert np.array_equal(out[:, rd:], x[:, rd:])  # dims past rotary_dim unchanged


def test_rotate_interleaved_is_split_on_permuted_dims():
    D, rd = 16, 16
    cos, sin, _ = _unit_angles(3, rd // 2, 4)
    x = np.random.default_rng(5).standard_normal((6, D))
    pos = np.array([0, 1, 2, 0, 1, 2])
    # interleaved pair j = (2j, 2j+1); split pair j = (j, j + rd/2)
    perm = np.concatenate([np.arange(0, rd, 2), np.arange(1, rd, 2)])
    a = orc.rotate(x, pos, cos, sin, rd, interleaved=True)
    b = orc.rotate(x[:, perm], pos, cos, sin, rd, interleaved=False)
    assert np.allclose(a[:, perm], b, rtol=0, atol=1e-12)


def test_rotate_invariants():
    D, rd = 8, 8
    # a Pythagorean angle: cos = 3/5, sin = 4/5 exactly; zero angle is the identity
    cos = np.array([[1.0] * 4, [0.6] * 4])
    sin = np.array([[0.0] * 4, [0.8] * 4])
    x = np.random.default_rng(6).standard_normal((2, D))
    pos = np.array([0, 1])
    for inter in (False, True):
        out = orc.rotate(x, pos, cos, sin, rd, interleaved=inter)
        assert np.array_equal(out[0], x[0])
        pairs_in = (x[1, 0::2], x[1, 1::2]) if inter else (x[1, :4], x[1, 4:])
        pairs_out = (out[1, 0::2], out[1, 1::2]) if inter else (out[1, :4], out[1, 4:])
        assert np.allclose(pairs_in[0] ** 2 + pairs_in[1] ** 2,
                           pairs_out[0] ** 2 + pairs_out[1] ** 2, rtol=1e-14, atol=0)
        back = orc.rotate(out, pos, cos, -sin, rd, interleaved=inter)
        assert np.allclose(back, x, rtol=0, atol=1e-14)


def test_rotary_write_uses_past_plus_index_and_packed_columns():
    # two sequences with different pasts; each position p rotates by the angle p * 0.1
    Hq, Hkv, D, P = 2, 1, 16, 16
    b = wl.ragged_batch([20, 9], [3, 9], Hq, Hkv, D, P, seed=64, poison=False)
    maxp = 32
    ang = 0.1 * np.arange(maxp)[:, None] * np.ones((1, D // 2))
    cos_b = _bf16_bits_from_f32(np.cos(ang).astype(np.float32))
    sin_b = _bf16_bits_from_f32(np.sin(ang).astype(np.float32))
    packed = torch.cat([b.q.reshape(b.num_tokens, -1), b.k_new.reshape(b.num_tokens, -1),
                        b.v_new.reshape(b.num_tokens, -1)], dim=1).contiguous()
    qo, kp, vp = orc.rotary_write_kv(packed, None, None, b.k_pool, b.v_pool, b.block_table,
                                     b.cu_seqlens_q, b.seq_lens_k, P, b.layout,
                                     num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                                     cos=cos_b, sin=sin_b, rotary_dim=D, interleaved=False)
    qo2, kp2, vp2 = orc.rotary_write_kv(b.q, b.k_new, b.v_new, b.k_pool, b.v_pool,
                                        b.block_table, b.cu_seqlens_q, b.seq_lens_k, P,
                                        b.layout, num_q_heads=Hq, num_kv_heads=Hkv,
                                        head_dim=D, cos=cos_b, sin=sin_b, rotary_dim=D)
    assert np.array_equal(qo, qo2) and np.array_equal(kp, kp2) and np.array_equal(vp, vp2)
    # token 1 of sequence 0 sits at position 17 + 1 = 18, token 0 of sequence 1 at 0
    cw, sw = orc.widen(cos_b), orc.widen(sin_b)
    for t, p in ((1, 18), (3, 0), (11, 8)):
        x = orc.widen(orc.bits16(b.q[t, 0]))
        z = (x[:D // 2] + 1j * x[D // 2:]) * (cw[p] + 1j * sw[p])
        want = orc.round_bf16(np.concatenate([z.real, z.imag]))
        assert np.array_equal(qo[t, 0], want)
    # V is scattered unchanged (the plain KV write of the same tokens)
    _, vref = orc.write_kv(b.k_pool, b.v_pool, b.k_new, b.v_new, b.block_table,
                           b.cu_seqlens_q, b.seq_lens_k, P, b.layout)
    assert np.array_equal(vp, vref)
    # without caches the pass is the plain split + scatter
    q3, kp3, _ = orc.rotary_write_kv(packed, None, None, b.k_pool, b.v_pool, b.block_table,
                                     b.cu_seqlens_q, b.seq_lens_k, P, b.layout,
                                     num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D)
    kref, _ = orc.write_kv(b.k_pool, b.v_pool, b.k_new, b.v_new, b.block_table,
                           b.cu_seqlens_q, b.seq_lens_k, P, b.layout)
    assert np.array_equal(q3, orc.bits16(b.q)) and np.array_equal(kp3, kref)


# --------------------------------------------------------------------------------------
# fp8 (e4m3) KV cache: the codec is pinned to the library's float8_e4m3fn conversions and to
# hand-derived values; the dequantised attention is pinned to the (already pinned) bf16
# oracle on values that both formats represent exactly.
# --------------------------------------------------------------------------------------

def test_e4m3_decode_matches_library_table():
    codes = np.arange(256, dtype=np.uint8)
    got = orc.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF]) and np.isnan(got).sum() == 2
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x38] == 1.0


def test_e4m3_encode_nearest_even_matches_library():
    rng = np.random.default_rng(71)
    vals = orc.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = (vals[1:] + vals[:-1]) / 2             # exact ties (representable in fp32)
    x = np.concatenate([rng.uniform(-447.9, 447.9, 50000), rng.normal(0, 0.05, 20000),
                        vals, -vals, mids, -mids]).astype(np.float32)
    got = orc.e4m3_encode(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("x,code", [
    (1.0, 0x38), (-1.0, 0xB8), (448.0, 0x7E), (500.0, 0x7E), (1e30, 0x7E), (-1e9, 0xFE),
    (2.0 ** -9, 0x01), (2.0 ** -10, 0x00), (1.5 * 2.0 ** -10, 0x01), (0.0, 0x00), (-0.0, 0x80),
    (1.0625, 0x38), (1.1875, 0x3A), (2.0 ** -6, 0x08), (7 * 2.0 ** -9, 0x07),
    (7.5 * 2.0 ** -9, 0x08), (float("nan"), 0x7F)])
def test_e4m3_encode_hand_values(x, code):
    # 1.0625 lies halfway between 1.0 (mantissa 000) and 1.125 (001): ties go to the even
    # mantissa; 1.1875 between 1.125 (001) and 1.25 (010) goes up; 2^-10 is half the
    # smallest subnormal and rounds to the even code 0; past 448 the code saturates.
    assert int(orc.e4m3_encode(np.array([x]))[0]) == code


def test_e4m3_round_trip_and_error_bound():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    v = orc.e4m3_decode(codes)
    back = orc.e4m3_encode(v)
    assert np.array_equal(orc.e4m3_decode(back), v)       # -0 and +0 both decode to 0
    rng = np.random.default_rng(72)
    x = rng.uniform(-440, 440, 20000)
    err = np.abs(orc.e4m3_decode(orc.e4m3_encode(x)) - x)
    # half a unit in the last place: 2^-4 relative for normals, 2^-10 absolute below 2^-6
    assert np.all(err <= np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10) * (1 + 1e-12))


def test_e4m3_quantize_divides_in_fp32_first():
    # 1.0 / 3.0 in fp32 is 0.3333333432674408; e4m3 neighbours 0.3125 and 0.34375
    bits = np.array([0x3F80], dtype=np.uint16)              # bf16 1.0
    code = orc.e4m3_quantize(bits, 3.0)
    assert orc.e4m3_decode(code)[0] == 0.34375
    # saturation: 2.0 / 2^-9 = 1024 -> 448
    assert int(orc.e4m3_quantize(bits * 0 + 0x4000, 2.0 ** -9)[0]) == 0x7E


@pytest.mark.parametrize("layout", [orc.SEQ_MAJOR, orc.HEAD_MAJOR])
def test_kv8_attention_equals_bf16_attention_on_shared_values(layout):
    b = wl.ragged_batch([70, 33, 129], [1, 3, 2], 8, 2, 128, 16, seed=81)
    if layout == orc.HEAD_MAJOR:
        b = wl.to_head_major(b)
    b8, _, _ = wl.with_kv8_pools(b, seed=82)
    # power-of-two scales keep code * scale exact in bf16: the e4m3 path must then give the
    # bf16 oracle's numbers on the same values, bit for bit
    ks = np.array([2.0 ** -5, 2.0 ** -3], dtype=np.float32)
    vs = np.array([2.0 ** -2, 2.0 ** 1], dtype=np.float32)
    kp8, vp8 = orc.codes8(b8.k_pool), orc.codes8(b8.v_pool)
    Hkv = 2

    def to_bf16(codes, scales):
        c = codes.copy()
        head_axis = 2 if layout == orc.SEQ_MAJOR else None
        v = orc.e4m3_decode(c)
        if head_axis is not None:
            v = v * scales.reshape(1, 1, Hkv, 1)
        else:  # head-major: page p belongs to one head; find it from the block table
            heads = np.zeros(c.shape[0], dtype=np.int64)
            bt = orc.ints(b8.block_table)
            for h in range(Hkv):
                heads[bt[:, h, :].reshape(-1)] = h
            v = v * scales[heads].reshape(-1, 1, 1)
        v = np.where(np.isnan(v), 0.0, v)
        return orc.round_bf16(v)

    # the step writes the new tokens (quantised) first; both sides then read the same
    # context and new-token values
    got_o, got_l, kpa, vpa = orc.forward_kv8(b8.q, b8.k_new, b8.v_new, kp8, vp8, ks, vs,
                                             b8.block_table, b8.cu_seqlens_q, b8.seq_lens_k,
                                             scale=b8.scale, causal=True, page_size=16,
                                             layout=layout)
    kb, vb = to_bf16(kpa, ks), to_bf16(vpa, vs)
    ref_o, ref_l = orc.attention(b8.q, kb, vb, b8.block_table, b8.cu_seqlens_q, b8.seq_lens_k,
                                 scale=b8.scale, causal=True, page_size=16, layout=layout,
                                 num_kv_heads=Hkv)
    assert np.all(np.isfinite(got_o))
    assert np.array_equal(got_o, ref_o) and np.array_equal(got_l, ref_l)


def test_kv8_attention_with_group_tables_equals_bf16_on_shared_values():
    # the e4m3 step restricted to a group table's blocks: the same numbers as the bf16
    # oracle with that table on the same (exactly shared) values, and not the dense result
    b = wl.to_head_major(wl.ragged_batch([600, 300], [100, 40], 8, 2, 128, 16, seed=85))
    b8, _, _ = wl.with_kv8_pools(b, seed=86)
    ks = np.array([2.0 ** -4, 2.0 ** -6], dtype=np.float32)
    vs = np.array([2.0 ** -1, 2.0 ** 0], dtype=np.float32)
    nqb, nkb = -(-100 // 16), b8.max_blocks
    # a group table is the union over its heads and query blocks: a low density keeps it sparse
    mask = wl.iid_block_mask(2, 8, nqb, nkb, seed=87, density=0.01)
    table, count = orc.build_group_tables(mask, 2)
    kp8, vp8 = orc.codes8(b8.k_pool), orc.codes8(b8.v_pool)
    got_o, got_l, kpa, vpa = orc.forward_kv8(b8.q, b8.k_new, b8.v_new, kp8, vp8, ks, vs,
                                             b8.block_table, b8.cu_seqlens_q, b8.seq_lens_k,
                                             scale=b8.scale, causal=True, page_size=16,
                                             layout=orc.HEAD_MAJOR, group_table=table,
                                             group_count=count)
    heads = np.zeros(kpa.shape[0], dtype=np.int64)
    bt = orc.ints(b8.block_table)
    for h in range(2):
        heads[bt[:, h, :].reshape(-1)] = h

    def to_bf16(codes, scales):
        v = orc.e4m3_decode(codes) * scales[heads].reshape(-1, 1, 1)
        return orc.round_bf16(np.where(np.isnan(v), 0.0, v))

    ref_o, ref_l = orc.attention(b8.q, to_bf16(kpa, ks), to_bf16(vpa, vs), b8.block_table,
                                 b8.cu_seqlens_q, b8.seq_lens_k, scale=b8.scale, causal=True,
                                 page_size=16, layout=orc.HEAD_MAJOR, num_kv_heads=2,
                                 group_table=table, group_count=count)
    assert np.array_equal(got_o, ref_o, equal_nan=True) and np.array_equal(got_l, ref_l,
                                                                           equal_nan=True)
    dense_o, _, _, _ = orc.forward_kv8(b8.q, b8.k_new, b8.v_new, kp8, vp8, ks, vs,
                                       b8.block_table, b8.cu_seqlens_q, b8.seq_lens_k,
                                       scale=b8.scale, causal=True, page_size=16,
                                       layout=orc.HEAD_MAJOR)
    fin = np.isfinite(got_o)
    assert fin.any() and not np.allclose(got_o[fin], dense_o[fin])


def test_write_kv8_places_quantised_codes_in_hand_derived_slots():
    b = wl.ragged_batch([5, 19], [2, 3], 4, 2, 128, 16, seed=83)
    b8, ks, vs = wl.with_kv8_pools(b, seed=84)
    kp, vp = orc.write_kv8(b8.k_pool, b8.v_pool, b8.k_new, b8.v_new, ks.numpy(), vs.numpy(),
                           b8.block_table, b8.cu_seqlens_q, b8.seq_lens_k, 16)
    bt = orc.ints(b8.block_table)
    # sequence 1: kv 19, q 3 -> positions 16, 17, 18 -> block 1, slots 0, 1, 2; tokens 2..4
    for i, pos in enumerate((16, 17, 18)):
        for h in range(2):
            want = orc.e4m3_quantize(orc.bits16(b8.k_new)[2 + i, h], float(ks[h]))
            assert np.array_equal(kp[bt[1, 1], pos % 16, h], want)
    # untouched slots keep their codes
    before = orc.codes8(b8.k_pool)
    mask = np.ones(before.shape[:2], dtype=bool)
    for (b_, pos) in [(0, 3), (0, 4), (1, 16), (1, 17), (1, 18)]:
        mask[bt[b_, pos // 16], pos % 16] = False
    assert np.array_equal(kp[mask], before[mask])


# --------------------------------------------------------------------------------------
# Per-(query tile, query head) tables: the block-sparse execution of the ablation
# --------------------------------------------------------------------------------------

def test_qtile_tables_hand_fixture():
    # B=1, Hq=2, 4 query blocks of 64 rows (two 128-row tiles), 6 KV blocks
    m = np.zeros((1, 2, 4, 6), dtype=np.uint8)
    m[0, 0, 0, [0, 3]] = 1      # head 0, tile 0 = q-blocks 0, 1
    m[0, 0, 1, [3, 5]] = 1
    m[0, 0, 3, [1]] = 1         # head 0, tile 1 = q-blocks 2, 3
    m[0, 1, 2, [2, 4]] = 1      # head 1: nothing in tile 0
    table, count = orc.build_qtile_tables(m, 64)
    assert table.shape == (1, 2, 2, 6)
    assert count.tolist() == [[[3, 1], [0, 2]]]
    assert table[0, 0, 0].tolist() == [0, 3, 5, -1, -1, -1]
    assert table[0, 0, 1].tolist() == [1, -1, -1, -1, -1, -1]
    assert table[0, 1, 0].tolist() == [-1] * 6
    assert table[0, 1, 1].tolist() == [2, 4, -1, -1, -1, -1]
    # q_block_rows 128: one query block per tile; 32: four per tile
    t1, c1 = orc.build_qtile_tables(m, 128)
    assert t1.shape == (1, 2, 4, 6) and c1[0, 0].tolist() == [2, 2, 0, 1]
    t4, c4 = orc.build_qtile_tables(m, 32)
    assert t4.shape == (1, 2, 1, 6) and c4[0].tolist() == [[4], [2]]


def _expand_union(table, count, Hq, nqb, nkb):
    """The unioned mask written back per (head, query block): every row of group g holds g's
    union (so block-sparse execution and per-group tables see the same blocks)."""
    B, Hkv = count.shape
    G = Hq // Hkv
    m = np.zeros((B, Hq, nqb, nkb), dtype=np.uint8)
    for b in range(B):
        for g in range(Hkv):
            sel = table[b, g, :count[b, g]]
            m[b, g * G:(g + 1) * G, :, sel] = 1
    return m


def test_qtile_tables_of_the_unioned_mask_equal_group_tables():
    rng = np.random.default_rng(61)
    mask = (rng.random((2, 8, 5, 23)) < 0.15).astype(np.uint8)
    gt, gc = orc.build_group_tables(mask, 2)
    u = _expand_union(gt, gc, 8, 5, 23)
    qt, qc = orc.build_qtile_tables(u, 64)
    for b in range(2):
        for hq in range(8):
            for tau in range(qt.shape[2]):
                assert qc[b, hq, tau] == gc[b, hq // 4]
                assert np.array_equal(qt[b, hq, tau], gt[b, hq // 4])


def test_qtile_attention_equals_group_attention_on_the_unioned_mask():
    P = 16
    b = wl.ragged_batch([300, 190], [260, 70], 8, 2, 32, P, seed=62, layout=wl.HEAD_MAJOR)
    nkb = b.max_blocks
    rng = np.random.default_rng(63)
    nqb = -(-260 // 64)
    mask = (rng.random((2, 8, nqb, nkb)) < 0.3).astype(np.uint8)
    gt, gc = orc.build_group_tables(mask, 2)
    o1, l1, _, _ = _oracle_forward(b, group_table=gt, group_count=gc)
    qt, qc = orc.build_qtile_tables(_expand_union(gt, gc, 8, nqb, nkb), 64)
    o2, l2, _, _ = _oracle_forward(b, qtile_table=qt, qtile_count=qc)
    assert np.array_equal(o1, o2, equal_nan=True) and np.array_equal(l1, l2, equal_nan=True)
    # a per-tile mask that differs between tiles and heads is not the union: rows of tile 0
    # of head 0 keep only block 0 -> attention over keys 0..15 of that row's prefix
    m2 = np.zeros_like(mask)
    m2[:, :, :, :] = 1
    m2[0, 0, :2, :] = 0
    m2[0, 0, :2, 0] = 1
    qt2, qc2 = orc.build_qtile_tables(m2, 64)
    o3, _, _, _ = _oracle_forward(b, qtile_table=qt2, qtile_count=qc2)
    past = 300 - 260
    for i in (0, 5, 127):
        n = min(past + i + 1, P)
        K = _f64(b.k_logical[0][:n, 0])
        V = _f64(b.v_logical[0][:n, 0])
        ref = _sdpa_row(_f64(b.q[i, 0]), K, V, b.scale)
        assert np.max(np.abs(o3[i, 0] - ref)) < 1e-12
    dense, _, _, _ = _oracle_forward(b)
    assert np.array_equal(o3[128:260, 0], dense[128:260, 0])   # tile 1: all blocks
    assert np.array_equal(o3[:, 1:], dense[:, 1:])


def test_kv8_output_check_rejects_a_dropped_decode_split():
    # The e4m3 attention check of the GPU tests must be able to fail.  Plant the mistake a
    # broken split-KV merge would make -- the last key split of two sequences lost (keys from
    # 256 of the 300-key sequence, from 768 of the 1025-key one) -- and require the check to
    # reject it, while the exact result rounded to bf16 passes.
    from tests.rpa_testing import kv8_output_errors, kv8_vmax
    b = wl.ragged_batch([1, 17, 300, 1025, 64], [1] * 5, 32, 8, 128, 16, seed=916)
    b8, ks, vs = wl.with_kv8_pools(b, seed=901)
    ref, _, kp, vp = orc.forward_kv8(b8.q, b8.k_new, b8.v_new, b8.k_pool, b8.v_pool,
                                     ks.numpy(), vs.numpy(), b8.block_table, b8.cu_seqlens_q,
                                     b8.seq_lens_k, scale=b8.scale, causal=True,
                                     page_size=16, layout=b8.layout)
    vmax = kv8_vmax(vp, vs.numpy())
    assert 1.0 < vmax < 10.0
    exact = torch.from_numpy(ref).to(torch.bfloat16)
    assert kv8_output_errors(exact, ref, vmax)[0]
    # attention of tokens 2 and 3 over their first split only (same pages, shorter context)
    cut, _ = orc.attention(b8.q, kp, vp, b8.block_table, b8.cu_seqlens_q,
                           np.array([1, 17, 256, 768, 64], dtype=np.int32), scale=b8.scale,
                           causal=True, page_size=16, layout=b8.layout, num_kv_heads=8,
                           rows=[(t, h) for t in (2, 3) for h in range(32)],
                           kv_scales=(ks.numpy(), vs.numpy()))
    mutated = ref.copy()
    mutated[2:4] = cut[2:4]
    ok, ratio, mean = kv8_output_errors(torch.from_numpy(mutated).to(torch.bfloat16), ref, vmax)
    assert not ok and ratio > 1.0 and mean > 2e-3, (ratio, mean)
