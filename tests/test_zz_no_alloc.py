"""rpa_forward_no_alloc: the fused step for callers that cannot allocate device memory (a
framework that owns every device byte, or a plugin interface that passes only inputs and
outputs).  Its scratch is the library's fixed per-device array, so its output must match the
entry point that takes a caller workspace, call after call.  This file is collected last."""
import numpy as np
import pytest
import torch

from ragged_paged_attention_forward_b200 import api
from ragged_paged_attention_forward_b200 import workloads as wl
from tests.rpa_testing import TOL_MAX, TOL_MEAN, plan_for, to_device

pytestmark = pytest.mark.gpu


def _run(batch, entry, plan):
    d = to_device(batch)
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


def test_no_alloc_matches_workspace_entry_point_on_consecutive_calls():
    # decode rows with several splits (partials + merge in the scratch) and a prefill row
    b = wl.ragged_batch([700, 1500, 2600, 300, 90], [1, 1, 1, 200, 3], 32, 8, 128, 16,
                        seed=71)
    plan = plan_for(b, decode_split_keys=256)
    info = plan.info()
    assert info.num_merge_rows > 0 and info.num_prefill_tiles > 0
    assert 0 < plan.workspace_bytes <= api.NO_ALLOC_WORKSPACE_BYTES
    ref_out, ref_lse = _run(b, "workspace", plan)
    for _ in range(2):
        out, lse = _run(b, "no_alloc", plan)
        err = (out.double() - ref_out.double()).abs()
        assert torch.isfinite(out.float()).all()
        assert err.max().item() <= TOL_MAX and err.mean().item() <= TOL_MEAN
        assert (lse - ref_lse).abs().max().item() <= 2e-3


def test_no_alloc_rejects_batches_beyond_its_scratch():
    b = wl.ragged_batch([4096] * 16, [1] * 16, 32, 8, 128, 16, seed=72, keep_logical=False)
    plan = plan_for(b, decode_split_keys=64)
    assert plan.workspace_bytes > api.NO_ALLOC_WORKSPACE_BYTES
    d = to_device(b)
    out = torch.empty_like(d["q"])
    with pytest.raises(api.RPAError) as ei:
        api.rpa_forward_no_alloc(plan, d["q"], d["k_new"], d["v_new"], d["k_pool"],
                                 d["v_pool"], d["block_table"], d["cu_seqlens_q"],
                                 d["seq_lens_k"], None, None, b.scale, out, None)
    assert ei.value.status == api.RPA_ERR_WORKSPACE_TOO_SMALL
    assert "built-in workspace" in str(ei.value)
