"""fp64 CPU oracle for ragged paged attention.  TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may import
this module.  It shares no code with the CUDA library and never imports it.

What it computes (plain definitions, written out; no tiling, no fusion, no reordering):

* ``write_kv``      -- the KV-cache scatter.  For token ``i`` of sequence ``b`` the absolute
  position is ``past_b + i`` with ``past_b = seq_lens_k[b] - q_len_b``; the page is
  ``block_table[b, pos // page_size]`` and the slot ``pos % page_size``.
  ([WebGPU] Optimized PagedAttention implementation (2/n), squashed commit "Phase 1b.1":
  ScatterKVToPagedCacheProgram index math.)
* ``attention``     -- exact softmax attention of every query row against the keys it may
  see, gathered through the block table.  Query ``i`` of sequence ``b`` sits at absolute
  position ``past_b + i`` and, when causal, sees keys ``0 .. past_b + i`` (bottom-right
  alignment: same page, commit "FlashAttention: optional seqlens_q input", which sets the
  per-batch past length to ``total_kv_b - seqlens_q[b]``).  Query head ``hq`` reads KV head
  ``hq // (Hq / Hkv)``.  With per-group block tables (CompactAttention: Accelerating
  Chunked Prefill with Block-Union KV Selection, Core claim and Fig. 3) only keys whose
  block is listed in the table of the row's KV group are visible.
  Output ``o = sum_j softmax_j(scale * q.k_j) v_j`` and ``lse = log sum_j exp(scale*q.k_j)``
  (natural log); a row that sees no key gets ``o = 0`` and ``lse = -inf``.
* ``merge_partials`` -- the log-sum-exp merge of attention over disjoint key sets (the
  split-reduce pair FlashAttentionPagedDecodeQKV / FlashAttentionPagedDecodeVxReduce of the
  WebGPU page, "What's shipped").
* ``build_group_tables`` -- Q-block union, then intra-group union, then the ascending list
  of selected KV blocks per (sequence, KV group) (CompactAttention, Core claim; Fig. 3).
* ``build_qtile_tables`` -- the per-(query tile, query head) lists of a block-sparse kernel
  that works per query block and head (CompactAttention, Fig. 7c: the execution-only
  ablation with the same unioned mask): row ``(b, hq, tile)`` lists, ascending, the KV blocks
  head ``hq`` selects in any query block of the 128-row tile.  ``attention`` with
  ``qtile_table`` lets row ``i`` of sequence ``b`` and head ``hq`` see only the blocks of
  its tile ``i // 128``.
* ``rotate`` / ``rotary_write_kv`` -- the input pass with rotary position embedding: Q and
  K rows rotated by their position ``past_b + s``, dims at or past ``rotary_dim`` unchanged,
  pairs interleaved ``(2j, 2j+1)`` or split ``(j, j + rotary_dim/2)``; a packed input holds
  per token the columns ``[Q | K | V]`` (same page, commits "Phase 1b.2" and the packed-QKV
  commit).  Each rotated value is the exact ``x1 c - x2 s`` / ``x1 s + x2 c`` rounded once to
  bf16 (nearest, ties to even).

* ``e4m3_decode`` / ``e4m3_encode`` / ``write_kv8`` / ``forward_kv8`` -- the fp8 KV cache
  (the quantised cache that the WebGPU page's commit "FlashAttention: optional seqlens_q
  input" defers under "Not in scope (deferred)").  A code is the e4m3 format written out:
  sign, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0 holds the subnormals
  ``m/8 * 2^-6``; ``S.1111.111`` is NaN; no infinities; the largest finite value is 448.
  Pool element = ``decode(code) * scale[kv head]``; a new element ``x`` is stored as the
  code nearest to ``fp32(x) / fp32(scale)`` (the quotient rounded once to fp32, then ties to
  the even code, magnitudes past 448 clamped to 448).  Plain reading of a silent page: the
  format and the rounding are the standard e4m3 ones; the per-KV-head scale is the plainest
  of the "per-page or per-head" choices.

Inputs are bf16 bit patterns (numpy ``uint16``) or torch bf16 tensors; every bf16 value is
widened exactly to fp64 before any arithmetic.  Cache writes move the bf16 bit patterns
unchanged.
"""
from __future__ import annotations

import math
from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np

SEQ_MAJOR = 0
HEAD_MAJOR = 1


# --------------------------------------------------------------------------------------
# bf16 handling
# --------------------------------------------------------------------------------------

def bits16(x) -> np.ndarray:
    """bf16 values as their uint16 bit patterns (a copy-free view where possible)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            assert x.dtype == torch.bfloat16, x.dtype
            return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    except ImportError:  # pragma: no cover
        pass
    x = np.asarray(x)
    assert x.dtype == np.uint16, x.dtype
    return x


def widen(bits: np.ndarray) -> np.ndarray:
    """Exact bf16 -> fp64: a bf16 is the top half of an IEEE fp32."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def ints(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().cpu().numpy().astype(np.int64)
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x).astype(np.int64)


# --------------------------------------------------------------------------------------
# Batch bookkeeping
# --------------------------------------------------------------------------------------

def seq_ranges(cu_seqlens_q, seq_lens_k) -> List[Tuple[int, int, int, int]]:
    """Per sequence: (first token, q_len, kv_len, past) with past = kv_len - q_len."""
    cu = ints(cu_seqlens_q)
    kv = ints(seq_lens_k)
    out = []
    for b in range(len(kv)):
        t0 = int(cu[b])
        q_len = int(cu[b + 1] - cu[b])
        kv_len = int(kv[b])
        out.append((t0, q_len, kv_len, kv_len - q_len))
    return out


def page_of(block_table: np.ndarray, layout: int, b: int, h: int, pos: np.ndarray,
            page_size: int) -> np.ndarray:
    """Physical page that holds absolute position ``pos`` of sequence ``b`` (KV head ``h``
    in the head-major layout)."""
    if layout == SEQ_MAJOR:
        return block_table[b, pos // page_size]
    return block_table[b, h, pos // page_size]


# --------------------------------------------------------------------------------------
# a2: KV write (scatter)
# --------------------------------------------------------------------------------------

def write_kv(k_pool, v_pool, k_new, v_new, block_table, cu_seqlens_q, seq_lens_k,
             page_size: int, layout: int = SEQ_MAJOR):
    """Return copies of the pools with every new token's K/V written into its slot."""
    kp = bits16(k_pool).copy()
    vp = bits16(v_pool).copy()
    kn = bits16(k_new)
    vn = bits16(v_new)
    bt = ints(block_table)
    num_kv_heads = kn.shape[1]
    for b, (t0, q_len, kv_len, past) in enumerate(seq_ranges(cu_seqlens_q, seq_lens_k)):
        for i in range(q_len):
            t = t0 + i
            pos = past + i
            slot = pos % page_size
            if layout == SEQ_MAJOR:
                page = bt[b, pos // page_size]
                kp[page, slot] = kn[t]
                vp[page, slot] = vn[t]
            else:
                for h in range(num_kv_heads):
                    page = bt[b, h, pos // page_size]
                    kp[page, slot] = kn[t, h]
                    vp[page, slot] = vn[t, h]
    return kp, vp


def logical_rows(pool, block_table, layout: int, b: int, h: int, n: int,
                 page_size: int) -> np.ndarray:
    """Keys (or values) ``0 .. n-1`` of sequence ``b``, KV head ``h``, gathered through the
    block table: uint16 ``[n, D]`` (bf16 pools) or uint8 ``[n, D]`` (e4m3 code pools)."""
    p = codes8(pool) if _is_codes8(pool) else bits16(pool)
    bt = ints(block_table)
    pos = np.arange(n, dtype=np.int64)
    pages = page_of(bt, layout, b, h, pos, page_size)
    slots = pos % page_size
    if layout == SEQ_MAJOR:
        return p[pages, slots, h]
    return p[pages, slots]


# --------------------------------------------------------------------------------------
# a3-a5, a8: attention
# --------------------------------------------------------------------------------------

def visible_keys(pos: int, kv_len: int, causal: bool, page_size: int,
                 selected_blocks: Optional[set]) -> np.ndarray:
    """Indices of the keys a query at absolute position ``pos`` may attend to."""
    hi = min(kv_len, pos + 1) if causal else kv_len
    j = np.arange(hi, dtype=np.int64)
    if selected_blocks is not None:
        blocks = np.fromiter(selected_blocks, dtype=np.int64, count=len(selected_blocks))
        j = j[np.isin(j // page_size, blocks)]
    return j


def attend_row(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float):
    """Softmax attention of one fp64 query row over fp64 keys/values (rows of K, V).

    Returns (o [D], lse).  With no keys: (0, -inf)."""
    if K.shape[0] == 0:
        return np.zeros(q.shape[0], dtype=np.float64), -math.inf
    s = scale * (K @ q)
    m = np.max(s)
    w = np.exp(s - m)
    z = np.sum(w)
    o = (w @ V) / z
    return o, float(m + math.log(z))


def attention(q, k_pool, v_pool, block_table, cu_seqlens_q, seq_lens_k, *, scale: float,
              causal: bool, page_size: int, layout: int = SEQ_MAJOR, num_kv_heads: int,
              group_table=None, group_count=None,
              rows: Optional[Iterable[Tuple[int, int]]] = None, kv_scales=None,
              qtile_table=None, qtile_count=None, tile_rows: int = 128):
    """Attention of every (token, query head) row -- or of ``rows`` only -- against the pools
    *as given* (call ``write_kv`` first for the fused semantics).  With ``kv_scales =
    (k_scale, v_scale)`` the pools hold e4m3 codes and key ``j`` of KV head ``h`` is
    ``e4m3_decode(code) * k_scale[h]`` (likewise V).

    Returns ``(out [T, Hq, D] fp64, lse [T, Hq] fp64)``; rows not computed are NaN.
    """
    qb = bits16(q)
    T, Hq, D = qb.shape
    Hkv = int(num_kv_heads)
    G = Hq // Hkv
    seqs = seq_ranges(cu_seqlens_q, seq_lens_k)
    gt = ints(group_table) if group_table is not None else None
    gc = ints(group_count) if group_count is not None else None
    qt = ints(qtile_table) if qtile_table is not None else None
    qc = ints(qtile_count) if qtile_count is not None else None

    out = np.full((T, Hq, D), np.nan, dtype=np.float64)
    lse = np.full((T, Hq), np.nan, dtype=np.float64)

    if rows is None:
        wanted = None
    else:
        wanted = {}
        for t, hq in rows:
            wanted.setdefault(int(t), set()).add(int(hq))

    for b, (t0, q_len, kv_len, past) in enumerate(seqs):
        if q_len == 0:
            continue
        toks = range(t0, t0 + q_len)
        if wanted is not None:
            toks = [t for t in toks if t in wanted]
            if not toks:
                continue
        for hk in range(Hkv):
            heads = [hk * G + g for g in range(G)]
            if wanted is not None and not any(h in wanted[t] for t in toks for h in heads):
                continue
            if kv_scales is None:
                K = widen(logical_rows(k_pool, block_table, layout, b, hk, kv_len, page_size))
                V = widen(logical_rows(v_pool, block_table, layout, b, hk, kv_len, page_size))
            else:
                ks, vs = (np.asarray(x, dtype=np.float32) for x in kv_scales)
                K = e4m3_decode(logical_rows(k_pool, block_table, layout, b, hk, kv_len,
                                             page_size)) * float(ks[hk])
                V = e4m3_decode(logical_rows(v_pool, block_table, layout, b, hk, kv_len,
                                             page_size)) * float(vs[hk])
            selected = None
            if gt is not None:
                selected = set(int(x) for x in gt[b, hk, :int(gc[b, hk])])
            for t in toks:
                pos = past + (t - t0)
                idx = visible_keys(pos, kv_len, causal, page_size, selected)
                for hq in heads:
                    if wanted is not None and hq not in wanted[t]:
                        continue
                    if qt is not None:   # this head's table for the row's query tile
                        tau = (t - t0) // tile_rows
                        sel = set(int(x) for x in qt[b, hq, tau, :int(qc[b, hq, tau])])
                        idx = visible_keys(pos, kv_len, causal, page_size, sel)
                    o, l = attend_row(widen(qb[t, hq]), K[idx], V[idx], scale)
                    out[t, hq] = o
                    lse[t, hq] = l
    return out, lse


def forward(q, k_new, v_new, k_pool, v_pool, block_table, cu_seqlens_q, seq_lens_k, *,
            scale: float, causal: bool, page_size: int, layout: int = SEQ_MAJOR,
            group_table=None, group_count=None, rows=None, qtile_table=None,
            qtile_count=None):
    """The fused step: write the new tokens' K/V into the pools, then attend.

    Returns ``(out, lse, k_pool_after, v_pool_after)``."""
    kp, vp = write_kv(k_pool, v_pool, k_new, v_new, block_table, cu_seqlens_q, seq_lens_k,
                      page_size, layout)
    num_kv_heads = bits16(k_new).shape[1]
    out, lse = attention(q, kp, vp, block_table, cu_seqlens_q, seq_lens_k, scale=scale,
                         causal=causal, page_size=page_size, layout=layout,
                         num_kv_heads=num_kv_heads, group_table=group_table,
                         group_count=group_count, rows=rows, qtile_table=qtile_table,
                         qtile_count=qtile_count)
    return out, lse, kp, vp


# --------------------------------------------------------------------------------------
# a4: log-sum-exp merge of partial results
# --------------------------------------------------------------------------------------

def merge_partials(parts: Sequence[Tuple[np.ndarray, float]]):
    """Combine attention results over disjoint key sets: ``M = max lse_i``,
    ``w_i = exp(lse_i - M)``, ``o = sum w_i o_i / sum w_i``, ``lse = M + log sum w_i``."""
    lses = np.array([p[1] for p in parts], dtype=np.float64)
    if np.all(np.isneginf(lses)):
        return np.zeros_like(parts[0][0]), -math.inf
    M = np.max(lses)
    w = np.exp(lses - M)
    o = sum(wi * p[0] for wi, p in zip(w, parts)) / np.sum(w)
    return o, float(M + math.log(np.sum(w)))


# --------------------------------------------------------------------------------------
# a7: block-union tables
# --------------------------------------------------------------------------------------

def build_group_tables(mask, num_kv_heads: int):
    """Per-(sequence, KV group) tables of selected KV blocks.

    Step 1 (Q-block union): a query head needs KV block ``kb`` if any of its query blocks
    selects it.  Step 2 (intra-group union): a KV group needs ``kb`` if any query head of the
    group needs it; query head ``hq`` belongs to group ``hq // (Hq / Hkv)``.  Step 3: list the
    needed blocks in ascending order.

    ``mask`` is uint8 ``[B, Hq, nqb, nkb]``.  Returns ``(table int32 [B, Hkv, nkb],
    count int32 [B, Hkv])``; table entries past ``count`` are -1.
    """
    m = np.asarray(mask.numpy() if hasattr(mask, "numpy") else mask).astype(np.uint8)
    B, Hq, nqb, nkb = m.shape
    Hkv = int(num_kv_heads)
    G = Hq // Hkv
    head_union = np.zeros((B, Hq, nkb), dtype=bool)
    for b in range(B):
        for hq in range(Hq):
            for qb in range(nqb):
                head_union[b, hq] |= m[b, hq, qb] != 0
    group_union = np.zeros((B, Hkv, nkb), dtype=bool)
    for b in range(B):
        for hq in range(Hq):
            group_union[b, hq // G] |= head_union[b, hq]
    table = np.full((B, Hkv, nkb), -1, dtype=np.int32)
    count = np.zeros((B, Hkv), dtype=np.int32)
    for b in range(B):
        for g in range(Hkv):
            sel = [kb for kb in range(nkb) if group_union[b, g, kb]]
            table[b, g, :len(sel)] = sel
            count[b, g] = len(sel)
    return table, count


def build_qtile_tables(mask, q_block_rows: int, tile_rows: int = 128):
    """Per (sequence, query head, query tile of ``tile_rows`` rows): the ascending KV blocks
    selected by any of the tile's query blocks.  Returns ``(table [B, Hq, nt, nkb] int32,
    -1 past the count; count [B, Hq, nt] int32)``."""
    m = np.asarray(mask.cpu().numpy() if hasattr(mask, "cpu") else mask) != 0
    B, Hq, nqb, nkb = m.shape
    per = tile_rows // q_block_rows
    nt = -(-nqb // per)
    table = np.full((B, Hq, nt, nkb), -1, dtype=np.int32)
    count = np.zeros((B, Hq, nt), dtype=np.int32)
    for b in range(B):
        for hq in range(Hq):
            for tau in range(nt):
                rows = m[b, hq, tau * per:(tau + 1) * per]
                sel = [kb for kb in range(nkb) if rows[:, kb].any()]
                table[b, hq, tau, :len(sel)] = sel
                count[b, hq, tau] = len(sel)
    return table, count


# --------------------------------------------------------------------------------------
# Rotary position embedding and the packed-QKV split (the input pass)
# --------------------------------------------------------------------------------------

def round_bf16(x) -> np.ndarray:
    """fp64 -> bf16 bit patterns, rounded once to nearest with ties to even (the plain
    definition: 8 significant bits; below 2^-126 the spacing is fixed at 2^-133)."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    flat = x.reshape(-1)
    res = out.reshape(-1)
    for i, v in enumerate(flat):
        if v != v:
            res[i] = 0x7FC0
            continue
        if v == 0.0 or math.isinf(v):
            res[i] = np.array([v], dtype=np.float32).view(np.uint32)[0] >> 16
            continue
        m, e = math.frexp(v)              # v = m * 2^e, 0.5 <= |m| < 1
        if e - 1 >= -126:                 # normal range: 8 significant bits
            r = math.ldexp(float(np.rint(math.ldexp(m, 8))), e - 8)
        else:                             # subnormal: multiples of 2^-133
            r = math.ldexp(float(np.rint(math.ldexp(v, 133))), -133)
        if abs(r) >= 2.0 ** 128:
            r = math.copysign(math.inf, r)
        res[i] = np.array([r], dtype=np.float32).view(np.uint32)[0] >> 16
    return out


def rotate(x: np.ndarray, pos, cos: np.ndarray, sin: np.ndarray, rotary_dim: int,
           interleaved: bool) -> np.ndarray:
    """Rotate the last axis of ``x`` (fp64 ``[..., D]``) by the angles of positions ``pos``
    (integers broadcast to ``x.shape[:-1]``); ``cos``/``sin`` are fp64 ``[max_pos, rd/2]``."""
    out = np.array(x, dtype=np.float64, copy=True)
    half = rotary_dim // 2
    c = cos[pos]
    s = sin[pos]
    if interleaved:
        x1 = out[..., 0:rotary_dim:2].copy()
        x2 = out[..., 1:rotary_dim:2].copy()
        out[..., 0:rotary_dim:2] = x1 * c - x2 * s
        out[..., 1:rotary_dim:2] = x1 * s + x2 * c
    else:
        x1 = out[..., :half].copy()
        x2 = out[..., half:rotary_dim].copy()
        out[..., :half] = x1 * c - x2 * s
        out[..., half:rotary_dim] = x1 * s + x2 * c
    return out


def split_packed(qkv, num_q_heads: int, num_kv_heads: int, head_dim: int):
    """Packed ``[T, (Hq + 2 Hkv) * D]`` bf16 bits -> Q ``[T, Hq, D]``, K, V ``[T, Hkv, D]``."""
    a = bits16(qkv)
    T = a.shape[0]
    a = a.reshape(T, -1)
    qd = num_q_heads * head_dim
    kd = num_kv_heads * head_dim
    return (a[:, :qd].reshape(T, num_q_heads, head_dim),
            a[:, qd:qd + kd].reshape(T, num_kv_heads, head_dim),
            a[:, qd + kd:qd + 2 * kd].reshape(T, num_kv_heads, head_dim))


def token_positions(cu_seqlens_q, seq_lens_k) -> np.ndarray:
    """Absolute position of every new token: ``past_b + i``."""
    cu = ints(cu_seqlens_q)
    out = np.zeros(int(cu[-1]), dtype=np.int64)
    for t0, q_len, kv_len, past in seq_ranges(cu_seqlens_q, seq_lens_k):
        out[t0:t0 + q_len] = past + np.arange(q_len)
    return out


def rotary_write_kv(q, k, v, k_pool, v_pool, block_table, cu_seqlens_q, seq_lens_k,
                    page_size: int, layout: int = SEQ_MAJOR, *, num_q_heads: int,
                    num_kv_heads: int, head_dim: int, cos=None, sin=None,
                    rotary_dim: int = 0, interleaved: bool = False):
    """The input pass: returns (q_out bits [T, Hq, D], k_pool bits, v_pool bits)."""
    if k is None:
        qb, kb, vb = split_packed(q, num_q_heads, num_kv_heads, head_dim)
    else:
        qb, kb, vb = bits16(q), bits16(k), bits16(v)
    if cos is not None:
        pos = token_positions(cu_seqlens_q, seq_lens_k)
        c = widen(bits16(cos))
        s_ = widen(bits16(sin))
        qb = round_bf16(rotate(widen(qb), pos[:, None], c, s_, rotary_dim, interleaved))
        kb = round_bf16(rotate(widen(kb), pos[:, None], c, s_, rotary_dim, interleaved))
    kp, vp = write_kv(k_pool, v_pool, kb, vb, block_table, cu_seqlens_q, seq_lens_k,
                      page_size, layout)
    return np.ascontiguousarray(qb), kp, vp


# --------------------------------------------------------------------------------------
# fp8 (e4m3) KV cache
# --------------------------------------------------------------------------------------

def _is_codes8(x) -> bool:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.dtype == torch.uint8
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x).dtype == np.uint8


def codes8(x) -> np.ndarray:
    """e4m3 codes as numpy ``uint8``."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            assert x.dtype == torch.uint8, x.dtype
            return x.detach().cpu().contiguous().numpy()
    except ImportError:  # pragma: no cover
        pass
    x = np.asarray(x)
    assert x.dtype == np.uint8, x.dtype
    return x


def e4m3_decode(codes) -> np.ndarray:
    """e4m3 codes -> fp64, from the format's fields (exact)."""
    c = codes8(codes).astype(np.int64)
    sign = np.where(c >> 7, -1.0, 1.0)
    e = (c >> 3) & 15
    m = (c & 7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & ((c & 7) == 7), np.nan, mag)
    return sign * mag


# the 127 non-negative finite codes in increasing order of value (code i has value
# _E4M3_VALUES[i]; consecutive codes are consecutive values)
_E4M3_VALUES = e4m3_decode(np.arange(0x7F, dtype=np.uint8))


def e4m3_encode(x) -> np.ndarray:
    """fp64 values (typically fp32 quotients) -> e4m3 codes: nearest value, ties to the even
    code (mantissa LSB 0), magnitudes at or past 448 clamped to 448, NaN -> 0x7F | sign."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    sign = np.signbit(x).astype(np.uint8) << np.uint8(7)
    hi = np.searchsorted(_E4M3_VALUES, np.minimum(a, 448.0), side="left")  # first >= a
    hi = np.clip(hi, 0, 0x7E)
    lo = np.clip(hi - 1, 0, 0x7E)
    d_hi = _E4M3_VALUES[hi] - a
    d_lo = a - _E4M3_VALUES[lo]
    pick_lo = (d_lo < d_hi) | ((d_lo == d_hi) & (lo % 2 == 0))
    code = np.where(pick_lo, lo, hi)
    code = np.where(a >= 448.0, 0x7E, code)
    code = np.where(np.isnan(x), 0x7F, code).astype(np.uint8)
    return code | sign


def e4m3_quantize(bits, scale: float) -> np.ndarray:
    """bf16 bit patterns -> codes of ``fp32(x) / fp32(scale)`` (one fp32 rounding, then the
    e4m3 rounding of ``e4m3_encode``)."""
    y = widen(bits).astype(np.float32) / np.float32(scale)
    return e4m3_encode(y.astype(np.float64))


def write_kv8(k_pool, v_pool, k_new, v_new, k_scale, v_scale, block_table, cu_seqlens_q,
              seq_lens_k, page_size: int, layout: int = SEQ_MAJOR):
    """``write_kv`` for e4m3 code pools: each new token's K/V row is quantised with its KV
    head's scale and stored in its slot.  Returns copies of the code pools."""
    kp = codes8(k_pool).copy()
    vp = codes8(v_pool).copy()
    kn = bits16(k_new)
    vn = bits16(v_new)
    ks = np.asarray(k_scale, dtype=np.float32)
    vs = np.asarray(v_scale, dtype=np.float32)
    bt = ints(block_table)
    num_kv_heads = kn.shape[1]
    for b, (t0, q_len, kv_len, past) in enumerate(seq_ranges(cu_seqlens_q, seq_lens_k)):
        for i in range(q_len):
            t = t0 + i
            pos = past + i
            slot = pos % page_size
            for h in range(num_kv_heads):
                page = bt[b, pos // page_size] if layout == SEQ_MAJOR else bt[b, h, pos // page_size]
                dst = (page, slot, h) if layout == SEQ_MAJOR else (page, slot)
                kp[dst] = e4m3_quantize(kn[t, h], float(ks[h]))
                vp[dst] = e4m3_quantize(vn[t, h], float(vs[h]))
    return kp, vp


def forward_kv8(q, k_new, v_new, k_pool, v_pool, k_scale, v_scale, block_table, cu_seqlens_q,
                seq_lens_k, *, scale: float, causal: bool, page_size: int,
                layout: int = SEQ_MAJOR, rows=None, group_table=None, group_count=None,
                qtile_table=None, qtile_count=None):
    """The fused step over e4m3 code pools: quantising write, then attention over the
    dequantised keys and values (restricted, as in ``attention``, to the blocks of the group
    or query-tile tables when given).  Returns ``(out, lse, k_pool_after, v_pool_after)``."""
    num_kv_heads = len(np.atleast_1d(k_scale))
    if k_new is not None:
        kp, vp = write_kv8(k_pool, v_pool, k_new, v_new, k_scale, v_scale, block_table,
                           cu_seqlens_q, seq_lens_k, page_size, layout)
    else:
        kp, vp = codes8(k_pool).copy(), codes8(v_pool).copy()
    out, lse = attention(q, kp, vp, block_table, cu_seqlens_q, seq_lens_k, scale=scale,
                         causal=causal, page_size=page_size, layout=layout,
                         num_kv_heads=num_kv_heads, rows=rows, kv_scales=(k_scale, v_scale),
                         group_table=group_table, group_count=group_count,
                         qtile_table=qtile_table, qtile_count=qtile_count)
    return out, lse, kp, vp
