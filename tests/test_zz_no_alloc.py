"""rpa_forward_no_alloc: the fused step for callers that cannot allocate device memory (a
framework that owns every device byte, or a plugin interface that passes only inputs and
outputs).  Its scratch is the library's fixed per-device array, which keeps what the previous
call left in it, so its output must equal -- bit for bit -- the output of the entry point
that takes a caller workspace, whatever ran before.  This file is collected last."""
import numpy as np
import pytest
import torch

from ragged_paged_attention_forward_b200 import api
from ragged_paged_attention_forward_b200 import workloads as wl
from tests.rpa_testing import assert_close, assert_lse_close, oracle_forward, plan_for, to_device

pytestmark = pytest.mark.gpu


def _run(batch, entry, plan, d=None):
    d = d if d is not None else to_device(batch)
    T, Hq, D = batch.q.shape
    out = torch.full((T, Hq, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((T, Hq), float("nan"), dtype=torch.float32, device="cuda")
    args = (plan, d["q"], d["k_new"], d["v_new"], d["k_pool"], d["v_pool"], d["block_table"],
            d["cu_seqlens_q"], d["seq_lens_k"], None, None, batch.scale, out, lse)
    if entry == "workspace":
        ws = torch.empty(max(plan.workspace_bytes, 256), dtype=torch.uint8, device="cuda")
        api.rpa_forward(*args, ws)
    else:
        api.rpa_forward_no_alloc(*args)
    torch.cuda.synchronize()
    assert api.rpa_device_error(clear=True) == 0
    return out.cpu(), lse.cpu()


def test_no_alloc_equals_workspace_entry_point_on_alternating_batches():
    # Two batches whose scratch differs in layout and size: A has decode rows cut into many
    # 256-key splits (long work lists, many partials and merge rows) and a prefill row; B has
    # other lengths, 1024-key splits (fewer items, fewer merge rows) and two prefill rows.
    # Running them alternately through the shared array leaves each call the other's stale
    # lists and partials; every no-alloc output must still equal the workspace output exactly.
    a = wl.ragged_batch([700, 1500, 2600, 300, 90], [1, 1, 1, 200, 3], 32, 8, 128, 16, seed=71)
    b = wl.ragged_batch([5000, 60, 1800, 400], [1, 1, 300, 130], 32, 8, 128, 16, seed=73)
    pa = plan_for(a, decode_split_keys=256)
    pb = plan_for(b, decode_split_keys=1024)
    ia, ib = pa.info(), pb.info()
    assert ia.num_merge_rows > ib.num_merge_rows > 0
    assert ia.num_decode_items != ib.num_decode_items and ib.num_prefill_tiles > 0
    cap = api.no_alloc_workspace_bytes()
    assert 0 < pb.workspace_bytes <= cap and 0 < pa.workspace_bytes <= cap
    want = {"a": _run(a, "workspace", pa), "b": _run(b, "workspace", pb)}
    for name in ("a", "b", "a", "b", "a"):
        batch, plan = (a, pa) if name == "a" else (b, pb)
        out, lse = _run(batch, "no_alloc", plan)
        assert torch.equal(out, want[name][0]), name
        assert torch.equal(lse, want[name][1]), name
    ref, ref_lse, _, _ = oracle_forward(a)
    assert_close(want["a"][0], ref)
    assert_lse_close(want["a"][1], ref_lse)


def test_no_alloc_device_planned_step():
    # a device-planned step (work lists built on the GPU inside the call) through the
    # built-in scratch, after the batches above left other contents in it
    B, HQ, HKV, D, P, MAX_T, MAX_KV = 4, 8, 2, 128, 16, 512, 2048
    b = wl.ragged_batch([1200, 300, 2048, 77], [1, 200, 1, 77], HQ, HKV, D, P, seed=75)
    plan = api.rpa_plan_device(num_seqs=B, max_tokens=MAX_T, num_q_heads=HQ,
                               num_kv_heads=HKV, head_dim=D, page_size=P,
                               num_pages=b.num_pages, max_blocks_per_seq=b.max_blocks,
                               layout=wl.SEQ_MAJOR, causal=True, max_kv_len=MAX_KV)
    assert plan.workspace_bytes <= api.no_alloc_workspace_bytes()
    T = b.num_tokens
    outs = []
    for entry in ("workspace", "no_alloc", "no_alloc"):
        d = to_device(b)
        z = lambda *s, dt=torch.bfloat16: torch.zeros(*s, dtype=dt, device="cuda")
        q, kn, vn = z(MAX_T, HQ, D), z(MAX_T, HKV, D), z(MAX_T, HKV, D)
        q[:T], kn[:T], vn[:T] = d["q"], d["k_new"], d["v_new"]
        out = torch.full((MAX_T, HQ, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((MAX_T, HQ), float("nan"), dtype=torch.float32, device="cuda")
        args = (plan, q, kn, vn, d["k_pool"], d["v_pool"], d["block_table"], d["cu_seqlens_q"],
                d["seq_lens_k"], None, None, b.scale, out, lse)
        if entry == "workspace":
            ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
            api.rpa_forward(*args, ws)
        else:
            api.rpa_forward_no_alloc(*args)
        torch.cuda.synchronize()
        assert api.rpa_device_error(clear=True) == 0
        outs.append((out[:T].cpu(), lse[:T].cpu()))
    for out, lse in outs[1:]:
        assert torch.equal(out, outs[0][0]) and torch.equal(lse, outs[0][1])
    ref, ref_lse, _, _ = oracle_forward(b)
    assert_close(outs[0][0], ref)
    assert_lse_close(outs[0][1], ref_lse)


def test_no_alloc_rejects_batches_beyond_its_scratch():
    b = wl.ragged_batch([4096] * 16, [1] * 16, 32, 8, 128, 16, seed=72, keep_logical=False)
    plan = plan_for(b, decode_split_keys=64)
    assert plan.workspace_bytes > api.no_alloc_workspace_bytes()
    d = to_device(b)
    out = torch.empty_like(d["q"])
    with pytest.raises(api.RPAError) as ei:
        api.rpa_forward_no_alloc(plan, d["q"], d["k_new"], d["v_new"], d["k_pool"],
                                 d["v_pool"], d["block_table"], d["cu_seqlens_q"],
                                 d["seq_lens_k"], None, None, b.scale, out, None)
    assert ei.value.status == api.RPA_ERR_WORKSPACE_TOO_SMALL
    assert "built-in workspace" in str(ei.value)
