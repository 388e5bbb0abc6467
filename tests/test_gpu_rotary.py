"""GPU parity of the input pass with rotary position embedding (rpa_rotary_write_kv) against
the fp64 oracle, through the C ABI: rotated queries and keys within one bf16 ulp of the
exactly rounded result (the kernel rounds an fp32 result), values and every slot that is
not written bit-exact; then attention on the rotated inputs."""
import math

import numpy as np
import pytest
import torch

from oracle import rpa_oracle as orc
from ragged_paged_attention_forward_b200 import api
from ragged_paged_attention_forward_b200 import workloads as wl
from tests.rpa_testing import assert_close, plan_for, to_device

pytestmark = pytest.mark.gpu


def _rope_caches(max_pos, rotary_dim, base=10000.0):
    """Standard RoPE angles p / base^(2j/rd) as bf16 [max_pos, rd/2] caches."""
    j = np.arange(rotary_dim // 2)
    ang = np.arange(max_pos)[:, None] / base ** (2.0 * j / rotary_dim)[None, :]
    cos = torch.tensor(np.cos(ang), dtype=torch.float32).to(torch.bfloat16)
    sin = torch.tensor(np.sin(ang), dtype=torch.float32).to(torch.bfloat16)
    return cos, sin


def _within_one_ulp(got_bits, want_bits, min_exact=0.99):
    if got_bits.size == 0:
        return
    g = orc.widen(got_bits.reshape(-1))
    w = orc.widen(want_bits.reshape(-1))
    exp = np.floor(np.log2(np.maximum(np.abs(w), 2.0 ** -126)))
    ulp = 2.0 ** (exp - 7)
    assert np.all(np.abs(g - w) <= ulp), f"max diff {np.max(np.abs(g - w) / ulp):.2f} ulp"
    exact = np.mean(got_bits.reshape(-1) == want_bits.reshape(-1))
    assert exact >= min_exact, f"only {exact:.4f} bit-exact"


def _run(b, *, packed, rotary_dim, interleaved, max_pos=None, d=None):
    T, Hq, D = b.q.shape
    Hkv = b.num_kv_heads
    plan = plan_for(b)
    d = d if d is not None else to_device(b)
    cos = sin = None
    if rotary_dim:
        max_pos = max_pos or int(b.seq_lens_k.max()) + 3
        cos, sin = _rope_caches(max_pos, rotary_dim)
    if packed:
        qin = torch.cat([d["q"].reshape(T, -1), d["k_new"].reshape(T, -1),
                         d["v_new"].reshape(T, -1)], dim=1).contiguous()
        kin = vin = None
    else:
        qin, kin, vin = d["q"], d["k_new"], d["v_new"]
    q_out = torch.full((T, Hq, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    api.rpa_rotary_write_kv(plan, qin, kin, vin, q_out, d["k_pool"], d["v_pool"],
                            d["block_table"], d["cu_seqlens_q"], d["seq_lens_k"],
                            cos.cuda() if cos is not None else None,
                            sin.cuda() if sin is not None else None, rotary_dim, interleaved)
    torch.cuda.synchronize()
    code = api.rpa_device_error(clear=True)
    want = orc.rotary_write_kv(qin.cpu() if packed else b.q, None if packed else b.k_new,
                               None if packed else b.v_new, b.k_pool, b.v_pool, b.block_table,
                               b.cu_seqlens_q, b.seq_lens_k, b.page_size, b.layout,
                               num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                               cos=cos, sin=sin, rotary_dim=rotary_dim,
                               interleaved=interleaved)
    return code, (orc.bits16(q_out.cpu()), orc.bits16(d["k_pool"].cpu()),
                  orc.bits16(d["v_pool"].cpu())), want, plan, d, q_out


@pytest.mark.parametrize("packed", [False, True])
@pytest.mark.parametrize("interleaved", [False, True])
@pytest.mark.parametrize("D,rd", [(128, 128), (128, 64), (64, 64), (64, 32)])
def test_rotary_write_matches_oracle(packed, interleaved, D, rd):
    b = wl.ragged_batch([700, 40, 1300], [300, 40, 1], 8, 2, D, 16, seed=70 + D + rd)
    code, (qo, kp, vp), (wq, wk, wv), *_ = _run(b, packed=packed, rotary_dim=rd,
                                                interleaved=interleaved)
    assert code == 0
    _within_one_ulp(qo, wq)
    # pools: the written K slots within an ulp, everything else (incl. NaN poison) bit-exact
    diff = kp != wk
    _within_one_ulp(kp[diff], wk[diff], min_exact=0.0)
    assert np.array_equal(vp, wv)


@pytest.mark.parametrize("layout", [wl.SEQ_MAJOR, wl.HEAD_MAJOR])
def test_no_rotation_is_a_bit_exact_split_and_scatter(layout):
    b = wl.ragged_batch([500, 64], [200, 64], 8, 2, 128, 32, seed=75, layout=layout)
    code, (qo, kp, vp), (wq, wk, wv), *_ = _run(b, packed=True, rotary_dim=0,
                                                interleaved=False)
    assert code == 0
    assert np.array_equal(qo, wq) and np.array_equal(kp, wk) and np.array_equal(vp, wv)


def test_head_major_rotation():
    b = wl.ragged_batch([300, 129], [150, 129], 8, 2, 128, 64, seed=76, layout=wl.HEAD_MAJOR)
    code, (qo, kp, vp), (wq, wk, wv), *_ = _run(b, packed=False, rotary_dim=128,
                                                interleaved=False)
    assert code == 0
    _within_one_ulp(qo, wq)
    diff = kp != wk
    _within_one_ulp(kp[diff], wk[diff], min_exact=0.0)
    assert np.array_equal(vp, wv)


def test_attention_on_rotated_inputs():
    # the input pass, then the fused step with the new K/V already in the cache
    b = wl.ragged_batch([900, 2000, 33], [400, 1, 33], 8, 2, 128, 16, seed=77)
    code, (qo, kp, vp), (wq, wk, wv), plan, d, q_out = _run(b, packed=True, rotary_dim=128,
                                                            interleaved=False)
    assert code == 0
    out = torch.empty_like(q_out)
    lse = torch.empty(b.num_tokens, b.num_q_heads, dtype=torch.float32, device="cuda")
    ws = torch.empty(max(plan.workspace_bytes, 256), dtype=torch.uint8, device="cuda")
    api.rpa_forward(plan, q_out, None, None, d["k_pool"], d["v_pool"], d["block_table"],
                    d["cu_seqlens_q"], d["seq_lens_k"], None, None, b.scale, out, lse, ws)
    torch.cuda.synchronize()
    assert api.rpa_device_error(clear=True) == 0
    ref, _ = orc.attention(wq, wk, wv, b.block_table, b.cu_seqlens_q, b.seq_lens_k,
                           scale=b.scale, causal=b.causal, page_size=b.page_size,
                           layout=b.layout, num_kv_heads=b.num_kv_heads)
    assert_close(out.cpu(), ref)


def test_position_past_the_caches_is_reported_and_not_written():
    b = wl.ragged_batch([100, 50], [10, 50], 8, 2, 128, 16, seed=78)
    d = to_device(b)
    q_before = torch.full_like(d["q"], 0.0)
    k_before = d["k_pool"].clone()
    plan = plan_for(b)
    cos, sin = _rope_caches(64, 128)  # sequence 0 reaches position 99
    q_out = q_before.clone()
    api.rpa_rotary_write_kv(plan, d["q"], d["k_new"], d["v_new"], q_out, d["k_pool"],
                            d["v_pool"], d["block_table"], d["cu_seqlens_q"], d["seq_lens_k"],
                            cos.cuda(), sin.cuda(), 128, False)
    torch.cuda.synchronize()
    assert api.rpa_device_error(clear=True) & 8
    # sequence 0's tokens (positions 90..99) are untouched in q_out and in the K pool
    assert torch.equal(q_out[:10], q_before[:10])
    pos = np.arange(90, 100)
    for p in pos:
        page = int(b.block_table[0, p // 16])
        assert torch.equal(d["k_pool"][page, p % 16].view(torch.int16),
                           k_before[page, p % 16].view(torch.int16))
