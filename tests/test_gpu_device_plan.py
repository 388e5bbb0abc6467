"""GPU parity of device-planned steps (rpa_plan_device): the work lists are built on the
device from the step's device lengths, so one captured CUDA graph serves batches of any
lengths within the plan's limits.  Compared with the fp64 oracle through the C ABI."""
import numpy as np
import pytest
import torch

from oracle import rpa_oracle as orc
from ragged_paged_attention_forward_b200 import api
from ragged_paged_attention_forward_b200 import workloads as wl
from tests.rpa_testing import (assert_close, assert_kv8_close, assert_lse_close, kv8_vmax,
                               oracle_forward)

pytestmark = pytest.mark.gpu

B, HQ, HKV, D, P = 6, 8, 2, 128, 16
MAX_T, MAX_KV, MAX_BLOCKS, NUM_PAGES = 1024, 4096, 4096 // 16, 2200


def _batch(kv_lens, q_lens, seed):
    b = wl.ragged_batch(kv_lens, q_lens, HQ, HKV, D, P, seed=seed, min_pages=NUM_PAGES,
                        pool_slack=1.0, extra_pages=1)
    assert b.num_pages == NUM_PAGES and b.max_blocks <= MAX_BLOCKS
    return b


class Step:
    """Fixed device buffers sized for the plan's limits, as a captured graph needs them."""

    def __init__(self, causal=True):
        self.plan = api.rpa_plan_device(num_seqs=B, max_tokens=MAX_T, num_q_heads=HQ,
                                        num_kv_heads=HKV, head_dim=D, page_size=P,
                                        num_pages=NUM_PAGES, max_blocks_per_seq=MAX_BLOCKS,
                                        layout=wl.SEQ_MAJOR, causal=causal, max_kv_len=MAX_KV)
        z = lambda *s, dt=torch.bfloat16: torch.zeros(*s, dtype=dt, device="cuda")
        self.q, self.out = z(MAX_T, HQ, D), z(MAX_T, HQ, D)
        self.k_new, self.v_new = z(MAX_T, HKV, D), z(MAX_T, HKV, D)
        self.lse = z(MAX_T, HQ, dt=torch.float32)
        self.k_pool, self.v_pool = z(NUM_PAGES, P, HKV, D), z(NUM_PAGES, P, HKV, D)
        self.bt = z(B, MAX_BLOCKS, dt=torch.int32)
        self.cu, self.kv = z(B + 1, dt=torch.int32), z(B, dt=torch.int32)
        self.ws = torch.empty(self.plan.workspace_bytes, dtype=torch.uint8, device="cuda")

    def load(self, b):
        T = b.num_tokens
        self.q[:T].copy_(b.q)
        self.k_new[:T].copy_(b.k_new)
        self.v_new[:T].copy_(b.v_new)
        self.k_pool.copy_(b.k_pool)
        self.v_pool.copy_(b.v_pool)
        self.bt.zero_()
        self.bt[:, :b.max_blocks].copy_(b.block_table)
        self.cu.copy_(b.cu_seqlens_q)
        self.kv.copy_(b.seq_lens_k)
        self.out.fill_(float("nan"))

    def run(self, scale):
        api.rpa_forward(self.plan, self.q, self.k_new, self.v_new, self.k_pool, self.v_pool,
                        self.bt, self.cu, self.kv, None, None, scale, self.out, self.lse,
                        self.ws)

    def check(self, b):
        T = b.num_tokens
        ref, ref_lse, kp, vp = oracle_forward(b)
        assert_close(self.out[:T].cpu(), ref)
        assert_lse_close(self.lse[:T].cpu(), ref_lse)
        assert np.array_equal(orc.bits16(self.k_pool.cpu()), kp)
        assert np.array_equal(orc.bits16(self.v_pool.cpu()), vp)


BATCHES = [
    ([1200, 3000, 700, 64, 4096, 33], [1, 1, 1, 1, 1, 1]),            # decode only
    ([700, 1500, 300, 128, 900, 60], [300, 200, 300, 1, 0, 60]),       # prefill + decode
    ([4096, 2, 3000, 1000, 17, 512], [1, 2, 4, 500, 17, 0]),           # short multi-token rows
]


@pytest.mark.parametrize("idx", range(len(BATCHES)))
def test_device_plan_matches_oracle(idx):
    kv, ql = BATCHES[idx]
    b = _batch(kv, ql, seed=80 + idx)
    st = Step()
    st.load(b)
    st.run(b.scale)
    torch.cuda.synchronize()
    assert api.rpa_device_error(clear=True) == 0
    st.check(b)


def test_one_captured_graph_serves_batches_of_different_lengths():
    st = Step()
    first = _batch(*BATCHES[0], seed=90)
    st.load(first)
    st.run(first.scale)  # warm-up outside the capture: streams, events, attributes
    torch.cuda.synchronize()
    assert api.rpa_device_error(clear=True) == 0
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        st.run(first.scale)
    for i, (kv, ql) in enumerate(BATCHES[1:] + BATCHES[:1]):
        b = _batch(kv, ql, seed=91 + i)
        st.load(b)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        assert api.rpa_device_error(clear=True) == 0
        st.check(b)
    del g


def test_step_beyond_the_limits_is_reported():
    st = Step()
    b = _batch([700, 64, 64, 64, 64, 64], [100, 1, 1, 1, 1, 1], seed=95)
    st.load(b)
    st.kv[0] = MAX_KV + 1  # past the plan's max_kv_len
    st.run(b.scale)
    torch.cuda.synchronize()
    assert api.rpa_device_error(clear=True) & 16


def test_e4m3_device_plan_graph_replays_any_batch():
    # a CUDA graph of rpa_forward_kv8 with a device plan made with kv_e4m3, replayed over
    # decode, short multi-token and long-chunk batches: the decode kernel quantises its rows'
    # new tokens and reads the codes, the scatter kernel quantises the rest and the
    # tensor-core kernel converts its tiles of codes to f16 itself
    plan = api.rpa_plan_device(num_seqs=B, max_tokens=MAX_T, num_q_heads=HQ, num_kv_heads=HKV,
                               head_dim=D, page_size=P, num_pages=NUM_PAGES,
                               max_blocks_per_seq=MAX_BLOCKS, layout=wl.SEQ_MAJOR, causal=True,
                               max_kv_len=MAX_KV, kv_e4m3=True)
    assert plan.info().launches_forward == 5
    z = lambda *s, dt=torch.bfloat16: torch.zeros(*s, dtype=dt, device="cuda")
    q, out = z(MAX_T, HQ, D), z(MAX_T, HQ, D)
    k_new, v_new = z(MAX_T, HKV, D), z(MAX_T, HKV, D)
    lse = z(MAX_T, HQ, dt=torch.float32)
    kp = z(NUM_PAGES, P, HKV, D, dt=torch.uint8)
    vp = z(NUM_PAGES, P, HKV, D, dt=torch.uint8)
    bt, cu, kv = z(B, MAX_BLOCKS, dt=torch.int32), z(B + 1, dt=torch.int32), z(B, dt=torch.int32)
    ks, vs = z(HKV, dt=torch.float32), z(HKV, dt=torch.float32)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")

    def load(b8, k_scale, v_scale):
        T = b8.num_tokens
        q.zero_(); k_new.zero_(); v_new.zero_()
        q[:T].copy_(b8.q); k_new[:T].copy_(b8.k_new); v_new[:T].copy_(b8.v_new)
        kp.copy_(b8.k_pool); vp.copy_(b8.v_pool)
        bt.zero_(); bt[:, :b8.max_blocks].copy_(b8.block_table)
        cu.copy_(b8.cu_seqlens_q); kv.copy_(b8.seq_lens_k)
        ks.copy_(k_scale); vs.copy_(v_scale)

    def step():
        api.rpa_forward_kv8(plan, q, k_new, v_new, kp, vp, ks, vs, bt, cu, kv, 1.0 / D ** 0.5,
                            out, lse, ws)

    batches = [([40, 700, 1, 3000, 129, 64], [1] * 6, 301),
               ([2, 90, 1500, 33, 4000, 10], [2, 1, 2, 1, 2, 1], 302),
               ([300, 40, 1, 2100, 1, 900], [300, 1, 1, 500, 1, 64], 303)]
    first = True
    graph = None
    for kv_lens, q_lens, seed in batches:
        b = _batch(kv_lens, q_lens, seed)
        b8, k_scale, v_scale = wl.with_kv8_pools(b, seed=seed + 1)
        load(b8, k_scale, v_scale)
        if first:
            step(); torch.cuda.synchronize()
            load(b8, k_scale, v_scale)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                step()
            first = False
        graph.replay()
        torch.cuda.synchronize()
        assert api.rpa_device_error(clear=True) == 0
        T = b8.num_tokens
        ref, ref_lse, kp_ref, vp_ref = orc.forward_kv8(
            b8.q, b8.k_new, b8.v_new, b8.k_pool, b8.v_pool, k_scale.numpy(), v_scale.numpy(),
            b8.block_table, b8.cu_seqlens_q, b8.seq_lens_k, scale=1.0 / D ** 0.5, causal=True,
            page_size=P, layout=wl.SEQ_MAJOR)
        assert np.array_equal(kp.cpu().numpy(), kp_ref) and np.array_equal(vp.cpu().numpy(), vp_ref)
        vmax = kv8_vmax(vp_ref, v_scale.numpy(), b8.block_table, wl.SEQ_MAJOR)
        assert_kv8_close(out[:T].cpu(), ref, vmax)
        assert_lse_close(lse[:T].cpu(), ref_lse)
    del graph
