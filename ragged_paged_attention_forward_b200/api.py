"""ctypes binding of librpa.so (include/rpa.h).  Argument marshalling only: every step of the
computation runs in the library's CUDA kernels.

Tensors are torch tensors (device memory and streams come from PyTorch); host arrays may be
torch CPU tensors, numpy arrays or lists.  Failures raise ``RPAError`` carrying the status
code and the library's message.  The library is loaded on first use; if it has not been built
this raises -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librpa.so")

RPA_OK = 0
RPA_ERR_INVALID_ARG = -1
RPA_ERR_UNSUPPORTED = -2
RPA_ERR_SHAPE = -3
RPA_ERR_WORKSPACE_TOO_SMALL = -4
RPA_ERR_CUDA = -5
RPA_ERR_DEVICE_CHECK = -6

LAYOUT_SEQ_MAJOR = 0
LAYOUT_HEAD_MAJOR = 1

CLASS_AUTO, CLASS_DECODE, CLASS_PREFILL, CLASS_MIXED = 0, 1, 2, 3


class Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "num_seqs", "num_tokens", "num_q_heads", "num_kv_heads", "head_dim", "page_size",
        "num_pages", "max_blocks_per_seq", "layout", "causal")]


class PlanOptions(ctypes.Structure):
    _fields_ = [("force_class", ctypes.c_int32), ("decode_split_keys", ctypes.c_int32),
                ("sparse", ctypes.c_int32), ("kv_e4m3", ctypes.c_int32),
                ("wait_test_us", ctypes.c_int32), ("reserved", ctypes.c_int32 * 3)]


class PlanInfo(ctypes.Structure):
    _fields_ = [("batch_class", ctypes.c_int32), ("num_decode_items", ctypes.c_int32),
                ("num_prefill_tiles", ctypes.c_int32), ("num_merge_rows", ctypes.c_int32),
                ("launches_forward", ctypes.c_int32), ("launches_write", ctypes.c_int32),
                ("decode_split_keys", ctypes.c_int32), ("tensor_core_grid", ctypes.c_int32),
                ("workspace_bytes", ctypes.c_size_t)]


class RPAError(RuntimeError):
    def __init__(self, func: str, status: int, message: str):
        super().__init__(f"{func}: {status_string(status)}: {message}")
        self.status = status


class Rotary(ctypes.Structure):
    _fields_ = [("cos_cache", ctypes.c_void_p), ("sin_cache", ctypes.c_void_p),
                ("max_position", ctypes.c_int32), ("rotary_dim", ctypes.c_int32),
                ("interleaved", ctypes.c_int32), ("reserved", ctypes.c_int32)]


_lib = None

_P = ctypes.c_void_p
_I32P = ctypes.POINTER(ctypes.c_int32)


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m ragged_paged_attention_forward_b200.build_native`")
        L = ctypes.CDLL(LIB_PATH)
        L.rpa_plan.argtypes = [ctypes.POINTER(Shape), _I32P, _I32P, ctypes.POINTER(PlanOptions),
                               ctypes.POINTER(_P), ctypes.POINTER(ctypes.c_size_t)]
        L.rpa_plan.restype = ctypes.c_int
        L.rpa_plan_device.argtypes = [ctypes.POINTER(Shape), ctypes.c_int32,
                                      ctypes.POINTER(PlanOptions), ctypes.POINTER(_P),
                                      ctypes.POINTER(ctypes.c_size_t)]
        L.rpa_plan_device.restype = ctypes.c_int
        L.rpa_plan_get_info.argtypes = [_P, ctypes.POINTER(PlanInfo)]
        L.rpa_plan_get_info.restype = ctypes.c_int
        L.rpa_plan_destroy.argtypes = [_P]
        L.rpa_plan_destroy.restype = None
        L.rpa_write_kv.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
        L.rpa_write_kv.restype = ctypes.c_int
        L.rpa_forward.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_float,
                                  _P, _P, _P, ctypes.c_size_t, _P]
        L.rpa_forward.restype = ctypes.c_int
        L.rpa_write_kv8.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]
        L.rpa_write_kv8.restype = ctypes.c_int
        L.rpa_forward_kv8.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                      ctypes.c_float, _P, _P, _P, ctypes.c_size_t, _P]
        L.rpa_forward_kv8.restype = ctypes.c_int
        L.rpa_forward_no_alloc.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                           ctypes.c_float, _P, _P, _P]
        L.rpa_forward_no_alloc.restype = ctypes.c_int
        L.rpa_no_alloc_workspace_bytes.argtypes = []
        L.rpa_no_alloc_workspace_bytes.restype = ctypes.c_size_t
        L.rpa_rotary_write_kv.argtypes = [_P, _P, _P, _P, ctypes.POINTER(Rotary), _P, _P, _P,
                                          _P, _P, _P, _P]
        L.rpa_rotary_write_kv.restype = ctypes.c_int
        L.rpa_build_group_tables.argtypes = [_P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                             ctypes.c_int32, ctypes.c_int32, _P, _P, _P]
        L.rpa_build_group_tables.restype = ctypes.c_int
        L.rpa_build_qtile_tables.argtypes = [_P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                             ctypes.c_int32, ctypes.c_int32, _P, _P, _P]
        L.rpa_build_qtile_tables.restype = ctypes.c_int
        L.rpa_device_error.argtypes = [_I32P, ctypes.c_int32]
        L.rpa_device_error.restype = ctypes.c_int
        L.rpa_status_string.argtypes = [ctypes.c_int]
        L.rpa_status_string.restype = ctypes.c_char_p
        L.rpa_last_error.argtypes = []
        L.rpa_last_error.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().rpa_status_string(status).decode()


def last_error() -> str:
    return lib().rpa_last_error().decode()


def _check(func: str, status: int):
    if status != RPA_OK:
        raise RPAError(func, status, last_error())


def _host_i32(x):
    """A host int32 array for the C ABI: contiguous int32 CPU tensors and numpy arrays are
    passed by pointer (the returned object keeps them alive for the call)."""
    if isinstance(x, torch.Tensor):
        if x.device.type == "cpu" and x.dtype == torch.int32 and x.is_contiguous():
            return _Keep(x, ctypes.cast(ctypes.c_void_p(x.data_ptr()), _I32P))
        x = x.detach().cpu().to(torch.int32).tolist()
    else:
        try:
            import numpy as np
            if isinstance(x, np.ndarray) and x.dtype == np.int32 and x.flags.c_contiguous:
                return _Keep(x, x.ctypes.data_as(_I32P))
        except ImportError:  # pragma: no cover
            pass
        x = [int(v) for v in x]
    arr = (ctypes.c_int32 * max(1, len(x)))(*x)
    return _Keep(arr, ctypes.cast(arr, _I32P))


class _Keep:
    """A ctypes pointer argument that holds a reference to the buffer it points into."""

    def __init__(self, owner, ptr):
        self.owner = owner
        self._as_parameter_ = ptr


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


class Plan:
    """Owns an rpa_plan_t."""

    def __init__(self, handle: ctypes.c_void_p, workspace_bytes: int):
        self._h = handle
        self.workspace_bytes = int(workspace_bytes)

    @property
    def handle(self) -> ctypes.c_void_p:
        return self._h

    def info(self) -> PlanInfo:
        info = PlanInfo()
        _check("rpa_plan_get_info", lib().rpa_plan_get_info(self._h, ctypes.byref(info)))
        return info

    def close(self):
        if self._h is not None and self._h.value:
            lib().rpa_plan_destroy(self._h)
        self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def rpa_plan(*, num_seqs: int, num_tokens: int, num_q_heads: int, num_kv_heads: int,
             head_dim: int, page_size: int, num_pages: int, max_blocks_per_seq: int,
             layout: int, causal: bool, cu_seqlens_q, seq_lens_k, force_class: int = 0,
             decode_split_keys: int = 0, sparse=False, kv_e4m3: bool = False,
             wait_test_us: int = 0) -> Plan:
    """wait_test_us > 0 is for tests of the bounded device waits only (see include/rpa.h):
    the decode kernel then loads nothing and reports its waits running out."""
    shape = Shape(num_seqs, num_tokens, num_q_heads, num_kv_heads, head_dim, page_size,
                  num_pages, max_blocks_per_seq, layout, 1 if causal else 0)
    # sparse: False/0 none, True/1 per-group tables, 2 per-(query tile, query head) tables
    opts = PlanOptions(force_class, decode_split_keys, int(sparse), 1 if kv_e4m3 else 0,
                       int(wait_test_us))
    handle = ctypes.c_void_p()
    ws = ctypes.c_size_t(0)
    _check("rpa_plan", lib().rpa_plan(ctypes.byref(shape), _host_i32(cu_seqlens_q),
                                      _host_i32(seq_lens_k), ctypes.byref(opts),
                                      ctypes.byref(handle), ctypes.byref(ws)))
    return Plan(handle, ws.value)


def rpa_plan_device(*, num_seqs: int, max_tokens: int, num_q_heads: int, num_kv_heads: int,
                    head_dim: int, page_size: int, num_pages: int, max_blocks_per_seq: int,
                    layout: int, causal: bool, max_kv_len: int,
                    decode_split_keys: int = 0, kv_e4m3: bool = False) -> Plan:
    """A plan whose work lists are built on the device at every call (CUDA-graph friendly):
    B = num_seqs sequences, at most max_tokens new tokens and max_kv_len keys per step.  The
    q / k_new / v_new / out / lse buffers of the calls hold max_tokens rows.  kv_e4m3: for
    rpa_forward_kv8."""
    shape = Shape(num_seqs, max_tokens, num_q_heads, num_kv_heads, head_dim, page_size,
                  num_pages, max_blocks_per_seq, layout, 1 if causal else 0)
    opts = PlanOptions(0, decode_split_keys, 0, 1 if kv_e4m3 else 0)
    handle = ctypes.c_void_p()
    ws = ctypes.c_size_t(0)
    _check("rpa_plan_device", lib().rpa_plan_device(ctypes.byref(shape), int(max_kv_len),
                                                    ctypes.byref(opts), ctypes.byref(handle),
                                                    ctypes.byref(ws)))
    return Plan(handle, ws.value)


def rpa_write_kv(plan: Plan, k_new, v_new, k_pool, v_pool, block_table, cu_seqlens_q,
                 seq_lens_k, workspace=None, stream=None):
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("rpa_write_kv", lib().rpa_write_kv(
        plan.handle, _ptr(k_new), _ptr(v_new), _ptr(k_pool), _ptr(v_pool), _ptr(block_table),
        _ptr(cu_seqlens_q), _ptr(seq_lens_k), _ptr(workspace), nbytes, _stream(stream)))


def rpa_forward(plan: Plan, q, k_new, v_new, k_pool, v_pool, block_table, cu_seqlens_q,
                seq_lens_k, group_table, group_count, scale: float, out, lse, workspace,
                stream=None):
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("rpa_forward", lib().rpa_forward(
        plan.handle, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_pool), _ptr(v_pool),
        _ptr(block_table), _ptr(cu_seqlens_q), _ptr(seq_lens_k), _ptr(group_table),
        _ptr(group_count), ctypes.c_float(scale), _ptr(out), _ptr(lse), _ptr(workspace), nbytes,
        _stream(stream)))


def rpa_write_kv8(plan: Plan, k_new, v_new, k_pool, v_pool, k_scale, v_scale, block_table,
                  cu_seqlens_q, seq_lens_k, stream=None):
    """Quantise and scatter the new tokens into e4m3 (uint8) pools with per-KV-head
    scales."""
    _check("rpa_write_kv8", lib().rpa_write_kv8(
        plan.handle, _ptr(k_new), _ptr(v_new), _ptr(k_pool), _ptr(v_pool), _ptr(k_scale),
        _ptr(v_scale), _ptr(block_table), _ptr(cu_seqlens_q), _ptr(seq_lens_k),
        _stream(stream)))


def rpa_forward_kv8(plan: Plan, q, k_new, v_new, k_pool, v_pool, k_scale, v_scale,
                    block_table, cu_seqlens_q, seq_lens_k, scale: float, out, lse, workspace,
                    stream=None, group_table=None, group_count=None):
    """The fused step over e4m3 (uint8) K/V pools with fp32 per-KV-head scales
    k_scale, v_scale [Hkv] (head_dim 128); group_table / group_count for sparse plans.
    Plans with rows for the tensor-core kernel, and device plans, must be made with
    kv_e4m3=True; see include/rpa.h."""
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("rpa_forward_kv8", lib().rpa_forward_kv8(
        plan.handle, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_pool), _ptr(v_pool),
        _ptr(k_scale), _ptr(v_scale), _ptr(block_table), _ptr(cu_seqlens_q), _ptr(seq_lens_k),
        _ptr(group_table), _ptr(group_count), ctypes.c_float(scale), _ptr(out), _ptr(lse),
        _ptr(workspace), nbytes, _stream(stream)))


def no_alloc_workspace_bytes() -> int:
    """Size of rpa_forward_no_alloc's built-in scratch, as compiled into the library."""
    return int(lib().rpa_no_alloc_workspace_bytes())


def rpa_forward_no_alloc(plan: Plan, q, k_new, v_new, k_pool, v_pool, block_table,
                         cu_seqlens_q, seq_lens_k, group_table, group_count, scale: float, out,
                         lse, stream=None):
    """rpa_forward without a workspace argument, for callers that cannot allocate device
    memory: the scratch lives in the library's fixed per-device array (see include/rpa.h).
    Calls that overlap on the GPU share that array and must be serialised by the caller."""
    _check("rpa_forward_no_alloc", lib().rpa_forward_no_alloc(
        plan.handle, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_pool), _ptr(v_pool),
        _ptr(block_table), _ptr(cu_seqlens_q), _ptr(seq_lens_k), _ptr(group_table),
        _ptr(group_count), ctypes.c_float(scale), _ptr(out), _ptr(lse), _stream(stream)))


def rpa_rotary_write_kv(plan: Plan, q, k, v, q_out, k_pool, v_pool, block_table, cu_seqlens_q,
                        seq_lens_k, cos_cache=None, sin_cache=None, rotary_dim: int = 0,
                        interleaved: bool = False, stream=None):
    """Rotate Q and K by position (when cos/sin caches are given), write Q to q_out and
    scatter K, V into the pools.  k = v = None: q is the packed [T, (Hq + 2 Hkv) * D] input."""
    rot = None
    if cos_cache is not None:
        rot = Rotary(cos_cache.data_ptr(), sin_cache.data_ptr(), int(cos_cache.shape[0]),
                     int(rotary_dim or 2 * cos_cache.shape[1]), 1 if interleaved else 0, 0)
    _check("rpa_rotary_write_kv", lib().rpa_rotary_write_kv(
        plan.handle, _ptr(q), _ptr(k), _ptr(v), ctypes.byref(rot) if rot is not None else None,
        _ptr(q_out), _ptr(k_pool), _ptr(v_pool), _ptr(block_table), _ptr(cu_seqlens_q),
        _ptr(seq_lens_k), _stream(stream)))


def rpa_build_group_tables(mask, num_kv_heads: int, table, count, stream=None):
    B, Hq, nqb, nkb = mask.shape
    _check("rpa_build_group_tables", lib().rpa_build_group_tables(
        _ptr(mask), B, Hq, num_kv_heads, nqb, nkb, _ptr(table), _ptr(count), _stream(stream)))


def rpa_build_qtile_tables(mask, q_block_rows: int, table, count, stream=None):
    """Per-(query tile, query head) tables [B, Hq, ntiles, nkb] from a block mask
    [B, Hq, nqb, nkb] (block-sparse execution, for plans made with sparse=2)."""
    B, Hq, nqb, nkb = mask.shape
    _check("rpa_build_qtile_tables", lib().rpa_build_qtile_tables(
        _ptr(mask), B, Hq, nqb, nkb, int(q_block_rows), _ptr(table), _ptr(count),
        _stream(stream)))


def rpa_device_error(clear: bool = True) -> int:
    code = ctypes.c_int32(0)
    st = lib().rpa_device_error(ctypes.byref(code), 1 if clear else 0)
    if st not in (RPA_OK, RPA_ERR_DEVICE_CHECK):
        _check("rpa_device_error", st)
    return int(code.value)
