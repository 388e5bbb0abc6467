"""The C ABI on the host: the library loads, exports every entry point that include/rpa.h
declares, and rejects bad arguments before touching the device.  CPU only (no kernel runs:
every call here returns before its first CUDA call)."""
import ctypes
import os
import re

import pytest

from ragged_paged_attention_forward_b200 import api
from ragged_paged_attention_forward_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "rpa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(rpa_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_entry_point():
    names = _declared_functions()
    assert {"rpa_plan", "rpa_write_kv", "rpa_forward", "rpa_build_group_tables"} <= set(names)
    L = ctypes.CDLL(api.LIB_PATH)
    for n in names:
        assert hasattr(L, n), n


def test_no_alloc_scratch_size_matches_the_header():
    # the binding reads the size from the library; it must be the header's macro
    text = open(os.path.join(ROOT, "include", "rpa.h")).read()
    m = re.search(r"#define RPA_NO_ALLOC_WORKSPACE_BYTES \(\(size_t\)(\d+) << (\d+)\)", text)
    assert m, "macro not found"
    assert api.no_alloc_workspace_bytes() == int(m.group(1)) << int(m.group(2))


def _shape(**kw):
    s = dict(num_seqs=2, num_tokens=2, num_q_heads=32, num_kv_heads=8, head_dim=128,
             page_size=16, num_pages=100, max_blocks_per_seq=16, layout=0, causal=True,
             cu_seqlens_q=[0, 1, 2], seq_lens_k=[40, 200])
    s.update(kw)
    return s


@pytest.mark.parametrize("kw,status", [
    (dict(num_q_heads=30), api.RPA_ERR_SHAPE),
    (dict(head_dim=96), api.RPA_ERR_UNSUPPORTED),
    (dict(page_size=24), api.RPA_ERR_UNSUPPORTED),
    (dict(page_size=8), api.RPA_ERR_UNSUPPORTED),
    (dict(page_size=512), api.RPA_ERR_UNSUPPORTED),
    (dict(seq_lens_k=[0, 200]), api.RPA_ERR_SHAPE),                    # q_len > kv_len
    (dict(seq_lens_k=[40, 16 * 16 + 1]), api.RPA_ERR_SHAPE),           # too many pages
    (dict(cu_seqlens_q=[0, 2, 1]), api.RPA_ERR_SHAPE),                 # decreasing
    (dict(cu_seqlens_q=[1, 1, 2]), api.RPA_ERR_SHAPE),                 # cu[0] != 0
    (dict(num_tokens=3), api.RPA_ERR_SHAPE),                           # cu[B] != T
    (dict(layout=2), api.RPA_ERR_INVALID_ARG),
    (dict(num_pages=0), api.RPA_ERR_SHAPE),
    (dict(sparse=True), api.RPA_ERR_UNSUPPORTED),                      # sparse needs head-major
    (dict(decode_split_keys=100), api.RPA_ERR_INVALID_ARG),
    (dict(force_class=7), api.RPA_ERR_INVALID_ARG),
    (dict(wait_test_us=-1), api.RPA_ERR_INVALID_ARG),
    (dict(wait_test_us=1000001), api.RPA_ERR_INVALID_ARG),
])
def test_plan_rejects(kw, status):
    with pytest.raises(api.RPAError) as ei:
        api.rpa_plan(**_shape(**kw))
    assert ei.value.status == status
    assert api.last_error() != ""


def test_plan_classifies_and_sizes():
    dec = wl.decode(num_seqs=8, keep_logical=False)
    from tests.rpa_testing import plan_for
    p = plan_for(dec)
    info = p.info()
    assert info.batch_class == api.CLASS_DECODE
    assert info.num_prefill_tiles == 0 and info.num_decode_items >= 8
    assert info.workspace_bytes == p.workspace_bytes > 0
    split = info.decode_split_keys
    assert split % 64 == 0
    expect_items = sum(-(-kv // split) for kv in dec.kv_lens())
    assert info.num_decode_items == expect_items
    multi = sum(1 for kv in dec.kv_lens() if kv > split)
    assert info.num_merge_rows == multi
    assert info.launches_forward == 1 + (1 if multi else 0)   # decode (+ merge); write fused

    pf = wl.ragged_batch([300, 64], [300, 40], 8, 2, 64, 16, seed=1)
    info = plan_for(pf).info()
    assert info.batch_class == api.CLASS_PREFILL
    assert info.num_prefill_tiles == 3 + 1 and info.num_decode_items == 0

    mx = wl.ragged_batch([300, 64, 90], [300, 1, 3], 8, 2, 64, 16, seed=1)
    info = plan_for(mx).info()
    assert info.batch_class == api.CLASS_MIXED
    assert info.num_prefill_tiles == 3
    assert info.num_decode_items == 2    # q_len*G = 4 and 12 <= 16: decode kernel

    forced = plan_for(mx, force_class=api.CLASS_PREFILL).info()
    assert forced.num_decode_items == 0 and forced.num_prefill_tiles == 5


def test_mixed_batches_plan_an_sm_split_only_when_both_parts_are_large():
    from tests.rpa_testing import plan_for
    # the mixed workload: the decode rows' 1.7 GB and the chunks' 192 units balance, so the
    # tensor-core grid gets part of the SMs (the device is not visible here: 148 assumed)
    g = plan_for(wl.mixed()).info().tensor_core_grid
    assert 32 <= g <= 116
    # small or lopsided batches keep one CTA per unit
    small = wl.ragged_batch([16, 40, 300, 77, 1000], [16, 4, 300, 1, 33], 8, 2, 128, 16,
                            seed=1, keep_logical=False)
    assert plan_for(small).info().tensor_core_grid == 0
    assert plan_for(wl.prefill()).info().tensor_core_grid == 0
    assert plan_for(wl.decode(keep_logical=False)).info().tensor_core_grid == 0


def test_launch_counts_with_the_write_in_the_kernels():
    from tests.rpa_testing import plan_for
    # a batch of only long rows: scatter kernel + tensor-core kernel
    pf = wl.ragged_batch([300, 64], [300, 64], 8, 2, 64, 16, seed=1, keep_logical=False)
    assert plan_for(pf).info().launches_forward == 2
    # a mixed batch: both attention kernels write their own rows (tensor-core kernel, decode
    # kernel, merge), the chunk's past (64) a multiple of the TMA box height (16)
    mx = wl.ragged_batch([300, 1000, 96], [300, 1, 32], 8, 2, 64, 16, seed=1, keep_logical=False)
    assert plan_for(mx).info().launches_forward == 3
    # a past of 69 leaves new rows in a box with older keys: the scatter kernel runs for them
    st = wl.ragged_batch([300, 1000, 101], [300, 1, 32], 8, 2, 64, 16, seed=1, keep_logical=False)
    assert plan_for(st).info().launches_forward == 4
    # e4m3 plans keep the quantising scatter kernel (the tensor-core kernel reads the codes in
    # place: no other launch)
    mx8 = wl.ragged_batch([300, 1000, 96], [300, 1, 32], 8, 2, 128, 16, seed=1, keep_logical=False)
    assert plan_for(mx8, kv_e4m3=True).info().launches_forward == 4


def test_zero_tokens_is_a_no_op():
    p = api.rpa_plan(**_shape(num_seqs=2, num_tokens=0, cu_seqlens_q=[0, 0, 0]))
    fake = ctypes.c_void_p(1 << 20)
    L = api.lib()
    st = L.rpa_forward(p.handle, fake, None, None, fake, fake, fake, fake, fake, None, None,
                       ctypes.c_float(0.1), fake, None, None, 0, None)
    assert st == api.RPA_OK
    st = L.rpa_write_kv(p.handle, None, None, fake, fake, fake, fake, fake, None, 0, None)
    assert st == api.RPA_OK


def _forward_status(plan, **over):
    fake = 1 << 20
    args = dict(q=fake, k_new=fake, v_new=fake, k_pool=fake, v_pool=fake, bt=fake, cu=fake,
                kv=fake, gt=None, gc=None, scale=0.1, out=fake, lse=None, ws=fake,
                ws_bytes=plan.workspace_bytes)
    args.update(over)
    P = lambda v: None if v is None else ctypes.c_void_p(v)
    return api.lib().rpa_forward(plan.handle, P(args["q"]), P(args["k_new"]), P(args["v_new"]),
                                 P(args["k_pool"]), P(args["v_pool"]), P(args["bt"]),
                                 P(args["cu"]), P(args["kv"]), P(args["gt"]), P(args["gc"]),
                                 ctypes.c_float(args["scale"]), P(args["out"]), P(args["lse"]),
                                 P(args["ws"]), args["ws_bytes"], None)


@pytest.mark.parametrize("over,status", [
    (dict(q=None), api.RPA_ERR_INVALID_ARG),
    (dict(out=None), api.RPA_ERR_INVALID_ARG),
    (dict(k_pool=None), api.RPA_ERR_INVALID_ARG),
    (dict(q=(1 << 20) + 8), api.RPA_ERR_INVALID_ARG),          # misaligned
    (dict(v_new=None), api.RPA_ERR_INVALID_ARG),               # k_new without v_new
    (dict(gt=1 << 20, gc=1 << 20), api.RPA_ERR_INVALID_ARG),   # tables need head-major
    (dict(gt=1 << 20), api.RPA_ERR_INVALID_ARG),               # table without count
    (dict(ws_bytes=0), api.RPA_ERR_WORKSPACE_TOO_SMALL),
    (dict(ws=None), api.RPA_ERR_WORKSPACE_TOO_SMALL),
    (dict(ws=(1 << 20) + 16), api.RPA_ERR_INVALID_ARG),        # workspace not 256-aligned
    (dict(scale=float("inf")), api.RPA_ERR_INVALID_ARG),
])
def test_forward_rejects_on_host(over, status):
    p = api.rpa_plan(**_shape())
    assert _forward_status(p, **over) == status


def test_sparse_plan_requires_tables():
    p = api.rpa_plan(**_shape(layout=1, sparse=True))
    assert _forward_status(p) == api.RPA_ERR_INVALID_ARG          # tables missing
    p2 = api.rpa_plan(**_shape(layout=1))
    assert _forward_status(p2, gt=1 << 20, gc=1 << 20) == api.RPA_ERR_INVALID_ARG


def test_group_table_builder_rejects():
    L = api.lib()
    assert L.rpa_build_group_tables(None, 1, 6, 4, 1, 1, None, None, None) == api.RPA_ERR_SHAPE
    assert L.rpa_build_group_tables(None, 1, 4, 2, 1, 70000, None, None,
                                    None) == api.RPA_ERR_UNSUPPORTED
    assert L.rpa_build_group_tables(None, 0, 4, 2, 1, 4, None, None, None) == api.RPA_OK


def test_status_strings():
    for code in range(-6, 1):
        assert api.status_string(code).startswith("RPA_")


def _rotary_status(plan, rotary=None, **over):
    fake = 1 << 20
    args = dict(q=fake, k=3 << 20, v=5 << 20, q_out=7 << 24, k_pool=fake, v_pool=fake,
                bt=fake, cu=fake, kv=fake)
    args.update(over)
    P = lambda v: None if v is None else ctypes.c_void_p(v)
    rot = None
    if rotary is not None:
        r = dict(cos=9 << 20, sin=11 << 20, max_position=4096, rotary_dim=128, interleaved=0,
                 reserved=0)
        r.update(rotary)
        rot = api.Rotary(P(r["cos"]), P(r["sin"]), r["max_position"], r["rotary_dim"],
                         r["interleaved"], r["reserved"])
    return api.lib().rpa_rotary_write_kv(
        plan.handle, P(args["q"]), P(args["k"]), P(args["v"]),
        ctypes.byref(rot) if rot is not None else None, P(args["q_out"]), P(args["k_pool"]),
        P(args["v_pool"]), P(args["bt"]), P(args["cu"]), P(args["kv"]), None)


@pytest.mark.parametrize("over,rotary,status", [
    (dict(q=None), None, api.RPA_ERR_INVALID_ARG),
    (dict(q_out=None), None, api.RPA_ERR_INVALID_ARG),
    (dict(v=None), None, api.RPA_ERR_INVALID_ARG),                 # k without v
    (dict(q_out=(1 << 20) + 256), None, api.RPA_ERR_INVALID_ARG),  # q_out overlaps q
    (dict(q=(1 << 20) + 8), None, api.RPA_ERR_INVALID_ARG),        # misaligned
    (dict(k_pool=None), None, api.RPA_ERR_INVALID_ARG),
    ({}, dict(rotary_dim=24), api.RPA_ERR_UNSUPPORTED),
    ({}, dict(rotary_dim=256), api.RPA_ERR_UNSUPPORTED),
    ({}, dict(rotary_dim=0), api.RPA_ERR_UNSUPPORTED),
    ({}, dict(cos=None), api.RPA_ERR_INVALID_ARG),
    ({}, dict(sin=(11 << 20) + 4), api.RPA_ERR_INVALID_ARG),       # misaligned cache
    ({}, dict(max_position=0), api.RPA_ERR_INVALID_ARG),
    ({}, dict(interleaved=2), api.RPA_ERR_INVALID_ARG),
    ({}, dict(reserved=1), api.RPA_ERR_INVALID_ARG),
])
def test_rotary_write_rejects_on_host(over, rotary, status):
    p = api.rpa_plan(**_shape())
    assert _rotary_status(p, rotary, **over) == status


def test_rotary_write_zero_tokens_is_a_no_op():
    p = api.rpa_plan(**_shape(num_seqs=2, num_tokens=0, cu_seqlens_q=[0, 0, 0]))
    assert _rotary_status(p, dict()) == api.RPA_OK


def _device_plan(**kw):
    s = dict(num_seqs=4, max_tokens=512, num_q_heads=32, num_kv_heads=8, head_dim=128,
             page_size=16, num_pages=1000, max_blocks_per_seq=64, layout=0, causal=True,
             max_kv_len=1024)
    s.update(kw)
    return api.rpa_plan_device(**s)


def test_device_plan_sizes_its_workspace_for_the_limits():
    p = _device_plan()
    info = p.info()
    assert info.batch_class == api.CLASS_AUTO
    assert info.num_decode_items == 4 * (1024 // info.decode_split_keys)
    assert info.num_merge_rows == 512 and info.num_prefill_tiles == 512 // 128 + 4
    assert p.workspace_bytes >= info.num_decode_items * 32 and p.workspace_bytes % 256 == 0
    # a decode-heavy bound: 64 tokens over 64 sequences; a sequence reaches the tensor-core
    # kernel only with q_len * G > 8 (q_len >= 3 for G = 4), so at most 21 partial tiles
    d = _device_plan(num_seqs=64, max_tokens=64).info()
    assert d.num_prefill_tiles == 1 + 64 // 3
    g16 = _device_plan(num_seqs=64, max_tokens=64, num_q_heads=128).info()  # G = 16, NT = 2
    assert g16.num_prefill_tiles == 1 + 64 // 2


@pytest.mark.parametrize("kw,status", [
    (dict(max_kv_len=0), api.RPA_ERR_SHAPE),
    (dict(max_kv_len=64 * 16 + 1), api.RPA_ERR_SHAPE),
    (dict(head_dim=96), api.RPA_ERR_UNSUPPORTED),
    (dict(decode_split_keys=100), api.RPA_ERR_INVALID_ARG),
])
def test_device_plan_rejects(kw, status):
    with pytest.raises(api.RPAError) as e:
        _device_plan(**kw)
    assert e.value.status == status


def test_forward_kv8_rejects_before_any_device_work():
    # decode-only plan, head_dim 128: missing scales are an argument error
    plan = api.rpa_plan(**_shape())
    with pytest.raises(api.RPAError) as ei:
        api.rpa_forward_kv8(plan, None, None, None, None, None, None, None, None, None, None,
                            0.1, None, None, None, stream=0)
    assert ei.value.status == api.RPA_ERR_INVALID_ARG
    # a plan with a prefill row made without kv_e4m3 and a head_dim-64 plan are unsupported
    for kw in (dict(cu_seqlens_q=[0, 1, 200], num_tokens=200, seq_lens_k=[40, 200]),
               dict(head_dim=64)):
        plan = api.rpa_plan(**_shape(**kw))
        with pytest.raises(api.RPAError) as ei:
            api.rpa_forward_kv8(plan, None, None, None, None, None, None, None, None, None,
                                None, 0.1, None, None, None, stream=0)
        assert ei.value.status == api.RPA_ERR_UNSUPPORTED, kw


def test_kv_e4m3_plan_option():
    # the tensor-core kernel converts the codes itself: an e4m3 plan needs no more workspace
    # than a bf16 one, with or without tensor-core rows, and group tables are accepted
    for kw in (dict(cu_seqlens_q=[0, 1, 200], num_tokens=200, seq_lens_k=[40, 200]), {}):
        plain = api.rpa_plan(**_shape(**kw))
        e4 = api.rpa_plan(**_shape(**kw), kv_e4m3=True)
        assert e4.workspace_bytes == plain.workspace_bytes
        assert e4.info().launches_forward == plain.info().launches_forward
    api.rpa_plan(**_shape(layout=1, sparse=True), kv_e4m3=True)
    with pytest.raises(api.RPAError) as ei:
        api.rpa_plan(**_shape(head_dim=64), kv_e4m3=True)
    assert ei.value.status == api.RPA_ERR_UNSUPPORTED


def test_e4m3_device_plan_runs_both_kernel_families():
    # planner, quantising scatter and tensor-core kernel (side stream), decode (with the
    # quantising write of its rows) and merge, as for bf16 pools
    p = _device_plan(kv_e4m3=True)
    assert p.info().launches_forward == 5
    assert _device_plan().info().launches_forward == 5
    with pytest.raises(api.RPAError) as e:
        _device_plan(kv_e4m3=True, head_dim=64)
    assert e.value.status == api.RPA_ERR_UNSUPPORTED
    # e4m3 pools with a device plan made without the option are refused before device work
    with pytest.raises(api.RPAError) as ei:
        api.rpa_forward_kv8(_device_plan(), None, None, None, None, None, None, None, None,
                            None, None, 0.1, None, None, None, stream=0)
    assert ei.value.status == api.RPA_ERR_UNSUPPORTED


def test_plan_accepts_odd_group_sizes():
    # G = 3: three rows per token on the decode kernel; a 40-token row (120 rows) goes to the
    # tensor-core kernel, one query head per CTA
    p = api.rpa_plan(**_shape(num_q_heads=12, num_kv_heads=4))
    info = p.info()
    assert info.num_prefill_tiles == 0 and info.num_decode_items >= 2
    m = api.rpa_plan(**_shape(num_q_heads=12, num_kv_heads=4, num_tokens=41,
                              cu_seqlens_q=[0, 1, 41], seq_lens_k=[40, 200])).info()
    assert m.num_prefill_tiles == 1 and m.num_decode_items >= 1
