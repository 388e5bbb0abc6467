"""Helpers shared by the GPU tests: move a generated batch to the device, run it through the
C ABI (ragged_paged_attention_forward_b200.api), and compare with the fp64 oracle."""
from __future__ import annotations

import numpy as np
import torch

from oracle import rpa_oracle as orc
from ragged_paged_attention_forward_b200 import api

# Attention tolerance against the fp64 oracle (bf16 inputs, fp32 accumulation).
TOL_MAX = 2e-2
TOL_MEAN = 2e-3


def plan_for(batch, **opts) -> api.Plan:
    return api.rpa_plan(num_seqs=batch.num_seqs, num_tokens=batch.num_tokens,
                        num_q_heads=batch.num_q_heads, num_kv_heads=batch.num_kv_heads,
                        head_dim=batch.head_dim, page_size=batch.page_size,
                        num_pages=batch.num_pages, max_blocks_per_seq=batch.max_blocks,
                        layout=batch.layout, causal=batch.causal,
                        cu_seqlens_q=batch.cu_seqlens_q, seq_lens_k=batch.seq_lens_k, **opts)


def to_device(batch, device="cuda"):
    return {k: getattr(batch, k).to(device).contiguous() for k in (
        "q", "k_new", "v_new", "k_pool", "v_pool", "block_table", "cu_seqlens_q", "seq_lens_k")}


def run_forward(batch, *, fused=True, scale=None, with_lse=True, group_table=None,
                group_count=None, plan_opts=None, dev=None, repeat=1):
    """Write + attend through rpa_forward (or rpa_write_kv then rpa_forward when fused=False).
    Returns CPU tensors (out, lse, k_pool, v_pool)."""
    plan_opts = dict(plan_opts or {})
    if group_table is not None:
        plan_opts.setdefault("sparse", True)
    plan = plan_for(batch, **plan_opts)
    d = dev if dev is not None else to_device(batch)
    T, Hq, D = batch.q.shape
    out = torch.full((T, Hq, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((T, Hq), float("nan"), dtype=torch.float32, device="cuda") if with_lse else None
    ws = torch.empty(max(plan.workspace_bytes, 256), dtype=torch.uint8, device="cuda")
    scale = batch.scale if scale is None else scale
    gt = group_table.to("cuda") if group_table is not None else None
    gc = group_count.to("cuda") if group_count is not None else None
    for _ in range(repeat):
        if fused:
            api.rpa_forward(plan, d["q"], d["k_new"], d["v_new"], d["k_pool"], d["v_pool"],
                            d["block_table"], d["cu_seqlens_q"], d["seq_lens_k"], gt, gc, scale,
                            out, lse, ws)
        else:
            api.rpa_write_kv(plan, d["k_new"], d["v_new"], d["k_pool"], d["v_pool"],
                             d["block_table"], d["cu_seqlens_q"], d["seq_lens_k"])
            api.rpa_forward(plan, d["q"], None, None, d["k_pool"], d["v_pool"], d["block_table"],
                            d["cu_seqlens_q"], d["seq_lens_k"], gt, gc, scale, out, lse, ws)
    torch.cuda.synchronize()
    assert api.rpa_device_error(clear=True) == 0
    return (out.cpu(), lse.cpu() if lse is not None else None, d["k_pool"].cpu(),
            d["v_pool"].cpu(), plan)


def oracle_forward(batch, *, scale=None, group_table=None, group_count=None, rows=None):
    return orc.forward(batch.q, batch.k_new, batch.v_new, batch.k_pool, batch.v_pool,
                       batch.block_table, batch.cu_seqlens_q, batch.seq_lens_k,
                       scale=batch.scale if scale is None else scale, causal=batch.causal,
                       page_size=batch.page_size, layout=batch.layout,
                       group_table=group_table, group_count=group_count, rows=rows)


def attention_errors(out_gpu: torch.Tensor, out_ref: np.ndarray, rows=None):
    got = out_gpu.double().numpy()
    if rows is not None:
        idx_t = np.array([r[0] for r in rows])
        idx_h = np.array([r[1] for r in rows])
        got = got[idx_t, idx_h]
        ref = out_ref[idx_t, idx_h]
    else:
        ref = out_ref
    assert np.all(np.isfinite(got)), "non-finite output"
    err = np.abs(got - ref)
    return float(err.max()), float(err.mean())


def assert_close(out_gpu, out_ref, rows=None, tol_max=TOL_MAX, tol_mean=TOL_MEAN):
    mx, mean = attention_errors(out_gpu, out_ref, rows)
    assert mx <= tol_max and mean <= tol_mean, f"max {mx:.3e} mean {mean:.3e}"
    return mx, mean


def assert_lse_close(lse_gpu, lse_ref, rows=None, tol=2e-3):
    g = lse_gpu.double().numpy()
    if rows is not None:
        g = np.array([g[t, h] for t, h in rows])
        r = np.array([lse_ref[t, h] for t, h in rows])
    else:
        r = lse_ref
    both_inf = np.isneginf(g) & np.isneginf(r)
    d = np.abs(np.where(both_inf, 0.0, g) - np.where(both_inf, 0.0, r))
    assert np.all(np.isfinite(d)), "lse mismatch in -inf pattern"
    assert d.max() <= tol, f"lse max err {d.max():.3e}"


# ------------------------------------------------------------------ e4m3 (fp8) KV cache

def kv8_vmax(v_pool_codes, v_scale, block_table=None, layout=orc.SEQ_MAJOR) -> float:
    """The largest |V| an e4m3 V pool holds: per KV head, the largest finite code magnitude
    times that head's scale, maximised over the heads.  e4m3 magnitudes grow with the low
    seven bits of the code (0x7F is NaN), so a histogram of those bits finds each head's
    largest value.  A KV-head-major pool needs the block table to know which pages belong to
    which head."""
    codes = orc.codes8(v_pool_codes)
    vs = np.asarray(v_scale, dtype=np.float64)
    best = 0.0
    for h in range(len(vs)):
        if layout == orc.SEQ_MAJOR:
            c = codes[:, :, h, :]
        else:
            pages = np.unique(orc.ints(block_table)[:, h, :])
            c = codes[pages[(pages >= 0) & (pages < codes.shape[0])]]
        hist = np.bincount(c.ravel() & np.uint8(0x7F), minlength=128)
        hist[0x7F] = 0
        if hist.any():
            top = int(np.nonzero(hist)[0].max())
            best = max(best, float(orc.e4m3_decode(np.array([top], np.uint8))[0]) * vs[h])
    return best


def kv8_output_errors(out, ref, vmax, rows=None):
    """Check e4m3-cache attention against the fp64 oracle; returns (ok, max_ratio, mean_err).

    Error model.  Scores are exact: e4m3 -> f16 and bf16 -> f16 are exact conversions (q in
    f16's normal range; below it the f16 rounding is under 2^-25 absolute), f16 products are
    exact in fp32, and the fp32 sums over D = 128 terms add a relative error far below 2^-20.
    Both kernels round the probabilities to f16 before P.V (relative 2^-11; the normaliser l
    sums the unrounded values, and the probabilities that fall below f16's normal range add
    at most 2^-25 each against l >= 1) and the output to bf16 (relative 2^-9).  So a row's
    error is at most 2^-11 * sum_j w_j |v_j| + 2^-9 |o| <= 2^-11 * max|V| + 2^-9 |o|, plus
    fp32 noise.  The pointwise bound allowed is twice that, 2^-10 * max|V| + 2^-8 * |o|, with
    max|V| the largest value the batch's V pool actually holds after the write
    (``kv8_vmax``).  The rounding errors are independent from key to key, so they average
    out: the mean absolute error must also meet the bf16 tolerance's mean-abs criterion,
    TOL_MEAN."""
    got = out.double().numpy() if isinstance(out, torch.Tensor) else np.asarray(out, np.float64)
    if rows is not None:
        it = np.array([r[0] for r in rows])
        ih = np.array([r[1] for r in rows])
        got, ref = got[it, ih], ref[it, ih]
    if not np.all(np.isfinite(got)):
        return False, float("inf"), float("inf")
    err = np.abs(got - ref)
    bound = 2.0 ** -10 * vmax + 2.0 ** -8 * np.abs(ref)
    ratio = float((err / bound).max())
    mean = float(err.mean())
    return ratio <= 1.0 and mean <= TOL_MEAN, ratio, mean


def assert_kv8_close(out, ref, vmax, rows=None):
    ok, ratio, mean = kv8_output_errors(out, ref, vmax, rows)
    assert ok, f"e4m3 attention: worst err/bound {ratio:.3f}, mean err {mean:.3e}"
