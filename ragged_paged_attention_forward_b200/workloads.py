"""Seeded synthetic inputs for ragged paged attention.

This module draws the inputs that the tests, the benchmark and the oracle's pins share:
ragged batches (query lengths, context lengths), bf16 query/key/value values, page pools,
block tables and block masks.  It holds none of the attention arithmetic: it only draws
random values, assigns pages and converts one pool layout into the other.

Input recipe (the same for every consumer):
  * one ``torch.Generator`` seeded per batch; values are bf16 draws of N(0, 1);
  * each sequence first gets its *logical* key/value rows ``[kv_len, Hkv, D]``; the last
    ``q_len`` rows are the new tokens of this step (``k_new``/``v_new``), the rows before
    them are the context that already sits in the cache;
  * physical pages come from ``torch.randperm(num_pages)`` and are handed out in logical
    order; the pool holds ``ceil(1.1 * pages_used) + 8`` pages, the spare ones shuffled in;
  * cache slots that hold no context yet (the new tokens' slots, the tail of the last page,
    pages nobody uses) are filled with bf16 NaN for correctness runs ("poison") and with
    zeros for timing runs;
  * block-table entries past a sequence's last page point at an unused (NaN) page, so a
    kernel that reads past the end produces NaN instead of plausible numbers.

e4m3 (fp8) pools (``with_kv8_pools``): the same batch with its context rows replaced by
random finite e4m3 codes (sign uniform, exponent field uniform in 3..11, mantissa uniform:
magnitudes 2^-4 .. 2^4 * 1.875), every other slot holding the NaN code 0x7F for correctness
runs (0 for timing runs), and per-KV-head fp32 scales drawn uniform in [0.005, 0.02] for K
and [0.05, 0.2] for V (so bf16 N(0,1) new tokens land across the code range, the largest
ones saturating).

Layouts (the two page layouts of the CompactAttention page, Fig. 4):
  * sequence-major: pool ``[num_pages, page_size, Hkv, D]``, block_table ``[B, max_blocks]``;
  * KV-head-major: pool ``[num_pages, page_size, D]``, block_table ``[B, Hkv, max_blocks]``.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import torch

SEQ_MAJOR = 0
HEAD_MAJOR = 1

BF16_NAN_BITS = 0x7FC0


@dataclasses.dataclass
class Batch:
    """One step's inputs.  All tensors live on the CPU; pools are the state *before* the
    new tokens are written."""

    q: torch.Tensor                 # [T, Hq, D] bf16
    k_new: torch.Tensor             # [T, Hkv, D] bf16
    v_new: torch.Tensor             # [T, Hkv, D] bf16
    k_pool: torch.Tensor            # seq-major [N, P, Hkv, D] / head-major [N, P, D] bf16
    v_pool: torch.Tensor
    block_table: torch.Tensor       # int32 [B, max_blocks] / [B, Hkv, max_blocks]
    cu_seqlens_q: torch.Tensor      # int32 [B + 1]
    seq_lens_k: torch.Tensor        # int32 [B]
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    layout: int
    causal: bool
    scale: float
    k_logical: Optional[List[torch.Tensor]] = None   # per seq [kv_len, Hkv, D] bf16
    v_logical: Optional[List[torch.Tensor]] = None
    name: str = ""

    @property
    def num_seqs(self) -> int:
        return int(self.seq_lens_k.numel())

    @property
    def num_tokens(self) -> int:
        return int(self.q.shape[0])

    @property
    def num_pages(self) -> int:
        return int(self.k_pool.shape[0])

    @property
    def max_blocks(self) -> int:
        return int(self.block_table.shape[-1])

    def q_lens(self) -> List[int]:
        cu = self.cu_seqlens_q.tolist()
        return [cu[i + 1] - cu[i] for i in range(len(cu) - 1)]

    def kv_lens(self) -> List[int]:
        return self.seq_lens_k.tolist()


def _fill_value(poison: bool) -> float:
    return float("nan") if poison else 0.0


def _randn_bf16(g: torch.Generator, *shape) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def ragged_batch(kv_lens: Sequence[int], q_lens: Sequence[int], num_q_heads: int,
                 num_kv_heads: int, head_dim: int, page_size: int, *, seed: int,
                 layout: int = SEQ_MAJOR, causal: bool = True, scale: Optional[float] = None,
                 poison: bool = True, keep_logical: bool = True, pool_slack: float = 1.1,
                 extra_pages: int = 8, min_pages: int = 0, name: str = "") -> Batch:
    """Draw one ragged batch.

    ``kv_lens[b]`` is the context length *including* the ``q_lens[b]`` new tokens (the
    new tokens sit at the tail of the sequence).
    """
    B = len(kv_lens)
    assert len(q_lens) == B
    for kv, ql in zip(kv_lens, q_lens):
        assert 0 <= ql <= kv
    g = torch.Generator().manual_seed(int(seed))
    Hq, Hkv, D, P = num_q_heads, num_kv_heads, head_dim, page_size
    T = int(sum(q_lens))

    k_log, v_log = [], []
    for kv in kv_lens:
        k_log.append(_randn_bf16(g, kv, Hkv, D))
        v_log.append(_randn_bf16(g, kv, Hkv, D))
    q = _randn_bf16(g, T, Hq, D)

    cu = [0]
    for ql in q_lens:
        cu.append(cu[-1] + ql)
    k_new = torch.empty(T, Hkv, D, dtype=torch.bfloat16)
    v_new = torch.empty(T, Hkv, D, dtype=torch.bfloat16)
    for b, (kv, ql) in enumerate(zip(kv_lens, q_lens)):
        k_new[cu[b]:cu[b + 1]] = k_log[b][kv - ql:]
        v_new[cu[b]:cu[b + 1]] = v_log[b][kv - ql:]

    blocks = [math.ceil(kv / P) for kv in kv_lens]
    max_blocks = max(1, max(blocks) if blocks else 1)
    units = sum(blocks) * (Hkv if layout == HEAD_MAJOR else 1)
    num_pages = max(int(math.ceil(units * pool_slack)) + extra_pages, units + 1, min_pages)
    perm = torch.randperm(num_pages, generator=g).to(torch.int64)
    used = perm[:units]
    spare_page = int(perm[units].item())  # never handed out: stays poison / zero

    fill = _fill_value(poison)
    if layout == SEQ_MAJOR:
        k_pool = torch.full((num_pages, P, Hkv, D), fill, dtype=torch.bfloat16)
        v_pool = torch.full((num_pages, P, Hkv, D), fill, dtype=torch.bfloat16)
        bt = torch.full((B, max_blocks), spare_page, dtype=torch.int32)
    else:
        k_pool = torch.full((num_pages, P, D), fill, dtype=torch.bfloat16)
        v_pool = torch.full((num_pages, P, D), fill, dtype=torch.bfloat16)
        bt = torch.full((B, Hkv, max_blocks), spare_page, dtype=torch.int32)

    off = 0
    for b, (kv, ql) in enumerate(zip(kv_lens, q_lens)):
        nb = blocks[b]
        past = kv - ql
        if layout == SEQ_MAJOR:
            pages = used[off:off + nb]
            off += nb
            bt[b, :nb] = pages.to(torch.int32)
            if past > 0:
                pos = torch.arange(past)
                pg = pages[pos // P]
                sl = pos % P
                k_pool[pg, sl] = k_log[b][:past]
                v_pool[pg, sl] = v_log[b][:past]
        else:
            pages = used[off:off + nb * Hkv].view(Hkv, nb)
            off += nb * Hkv
            bt[b, :, :nb] = pages.to(torch.int32)
            if past > 0:
                pos = torch.arange(past)
                sl = pos % P
                for h in range(Hkv):
                    pg = pages[h][pos // P]
                    k_pool[pg, sl] = k_log[b][:past, h]
                    v_pool[pg, sl] = v_log[b][:past, h]

    if scale is None:
        scale = 1.0 / math.sqrt(D)
    return Batch(q=q, k_new=k_new, v_new=v_new, k_pool=k_pool, v_pool=v_pool,
                 block_table=bt, cu_seqlens_q=torch.tensor(cu, dtype=torch.int32),
                 seq_lens_k=torch.tensor(list(kv_lens), dtype=torch.int32),
                 num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D, page_size=P,
                 layout=layout, causal=causal, scale=float(scale),
                 k_logical=k_log if keep_logical else None,
                 v_logical=v_log if keep_logical else None, name=name)


def to_head_major(batch: Batch) -> Batch:
    """The same logical keys/values in the KV-head-major layout.

    Physical page ``p`` of the sequence-major pool becomes pages ``p*Hkv + h`` (one per KV
    head); the per-head table is ``block_table[b, j] * Hkv + h``.  This is a transpose of
    the pool, not a reshape.
    """
    assert batch.layout == SEQ_MAJOR
    N, P, Hkv, D = batch.k_pool.shape
    k_hm = batch.k_pool.permute(0, 2, 1, 3).reshape(N * Hkv, P, D).contiguous()
    v_hm = batch.v_pool.permute(0, 2, 1, 3).reshape(N * Hkv, P, D).contiguous()
    bt = batch.block_table.to(torch.int64)
    heads = torch.arange(Hkv, dtype=torch.int64).view(1, Hkv, 1)
    bt_hm = (bt.unsqueeze(1) * Hkv + heads).to(torch.int32).contiguous()
    return dataclasses.replace(batch, k_pool=k_hm, v_pool=v_hm, block_table=bt_hm,
                               layout=HEAD_MAJOR)


def permute_pages(batch: Batch, seed: int) -> Batch:
    """Move every physical page to a new random slot of the pool and rewrite the table to
    match.  The logical content of every sequence is unchanged."""
    g = torch.Generator().manual_seed(int(seed))
    N = batch.k_pool.shape[0]
    perm = torch.randperm(N, generator=g)        # old page i -> new page perm[i]
    k_new_pool = torch.empty_like(batch.k_pool)
    v_new_pool = torch.empty_like(batch.v_pool)
    k_new_pool[perm] = batch.k_pool
    v_new_pool[perm] = batch.v_pool
    bt = perm.to(torch.int32)[batch.block_table.to(torch.int64)]
    return dataclasses.replace(batch, k_pool=k_new_pool, v_pool=v_new_pool, block_table=bt)


# ---------------------------------------------------------------------------------------
# Block masks for the block-union tables (CompactAttention page, Sec. "Block-Union KV
# Selection"; Fig. 3).  The pages give no mask distribution; the recipe below keeps the
# per-group union near a quarter of the blocks instead of the near-dense union that an
# i.i.d. 25% mask would give after a 32-way OR.
# ---------------------------------------------------------------------------------------

def structured_block_mask(num_seqs: int, num_q_heads: int, num_kv_heads: int, nqb: int,
                          nkb: int, *, seed: int, past_blocks: int = 0,
                          group_density: float = 0.20, head_density: float = 0.02,
                          keep_prob: float = 0.5) -> torch.Tensor:
    """uint8 mask ``[B, Hq, nqb, nkb]``.

    Each KV group draws a base block set (``group_density``), each query head a private set
    (``head_density``); every (head, q-block) row keeps each block of the union of the two
    with probability ``keep_prob`` and always keeps block 0 and its own diagonal block
    ``past_blocks + qb`` (when that is < nkb).
    """
    g = torch.Generator().manual_seed(int(seed))
    Hq, Hkv = num_q_heads, num_kv_heads
    G = Hq // Hkv
    base = torch.rand(num_seqs, Hkv, nkb, generator=g) < group_density
    priv = torch.rand(num_seqs, Hq, nkb, generator=g) < head_density
    base_per_head = base.repeat_interleave(G, dim=1)
    cand = (base_per_head | priv).unsqueeze(2).expand(num_seqs, Hq, nqb, nkb)
    keep = torch.rand(num_seqs, Hq, nqb, nkb, generator=g) < keep_prob
    mask = cand & keep
    mask[..., 0] = True
    for qb in range(nqb):
        kb = past_blocks + qb
        if kb < nkb:
            mask[:, :, qb, kb] = True
    return mask.to(torch.uint8).contiguous()


def iid_block_mask(num_seqs: int, num_q_heads: int, nqb: int, nkb: int, *, seed: int,
                   density: float) -> torch.Tensor:
    g = torch.Generator().manual_seed(int(seed))
    return (torch.rand(num_seqs, num_q_heads, nqb, nkb, generator=g) < density).to(
        torch.uint8).contiguous()


# ---------------------------------------------------------------------------------------
# The five workloads.  Shapes are Llama-3-8B attention (32 query heads, 8 KV heads, head
# dim 128) except the tiny correctness case.  Seeds are 1000 + workload id.
# ---------------------------------------------------------------------------------------

def tiny(seed: int = 1001, poison: bool = True) -> Batch:
    """3 sequences, kv_len {17, 64, 130}, q_len {1, 1, 5} at the tail, Hq 4, Hkv 2, D 64,
    page 16, a 64-page pool in random order."""
    return ragged_batch([17, 64, 130], [1, 1, 5], 4, 2, 64, 16, seed=seed, poison=poison,
                        pool_slack=1.0, extra_pages=0, min_pages=64, name="tiny")


def decode(seed: int = 1002, poison: bool = True, num_seqs: int = 64,
           keep_logical: bool = True) -> Batch:
    """Decode only: ``num_seqs`` sequences with q_len 1 and kv_len ~ U[512, 8192]."""
    g = torch.Generator().manual_seed(int(seed) + 7919)
    kv = torch.randint(512, 8192 + 1, (num_seqs,), generator=g).tolist()
    return ragged_batch(kv, [1] * num_seqs, 32, 8, 128, 16, seed=seed, poison=poison,
                        keep_logical=keep_logical, name="decode")


def prefill(seed: int = 1003, poison: bool = True, num_seqs: int = 4, prompt: int = 4096,
            keep_logical: bool = True) -> Batch:
    """Prefill only: ``num_seqs`` prompts of ``prompt`` tokens, no earlier context, page 64."""
    return ragged_batch([prompt] * num_seqs, [prompt] * num_seqs, 32, 8, 128, 64,
                        seed=seed, poison=poison, keep_logical=keep_logical, name="prefill")


def mixed(seed: int = 1004, poison: bool = True, num_decode: int = 48,
          keep_logical: bool = True, shuffle: bool = False) -> Batch:
    """Continuous batch under a 2048-token budget: ``num_decode`` decode rows
    (kv_len ~ U[1024, 16384]) plus two prefill chunks of 512 and 976 tokens whose earlier
    context is 1024 and 8192 tokens; page 16."""
    g = torch.Generator().manual_seed(int(seed) + 7919)
    kv = torch.randint(1024, 16384 + 1, (num_decode,), generator=g).tolist()
    ql = [1] * num_decode
    kv += [1024 + 512, 8192 + 976]
    ql += [512, 976]
    if shuffle:
        order = torch.randperm(len(kv), generator=g).tolist()
        kv = [kv[i] for i in order]
        ql = [ql[i] for i in order]
    return ragged_batch(kv, ql, 32, 8, 128, 16, seed=seed, poison=poison,
                        keep_logical=keep_logical, name="mixed")


SPARSE_BLOCK = 64


def sparse(seed: int = 1005, poison: bool = True, kv_len: int = 131072, chunk: int = 2048,
           keep_logical: bool = False):
    """Sparse chunked prefill: one sequence, a ``chunk``-token query chunk at the end of a
    ``kv_len`` context, KV-head-major pages of 64, and a per-head 64x64 block mask.

    Returns ``(batch, mask)``; mask is uint8 ``[1, 32, chunk/64, kv_len/64]``.
    """
    batch = ragged_batch([kv_len], [chunk], 32, 8, 128, SPARSE_BLOCK, seed=seed,
                         layout=HEAD_MAJOR, poison=poison, keep_logical=keep_logical,
                         name="sparse")
    return batch, sparse_mask(seed=seed, kv_len=kv_len, chunk=chunk)


def sparse_mask(seed: int = 1005, kv_len: int = 131072, chunk: int = 2048) -> torch.Tensor:
    """The block mask of the sparse chunked-prefill workload alone."""
    nqb = chunk // SPARSE_BLOCK
    nkb = math.ceil(kv_len / SPARSE_BLOCK)
    return structured_block_mask(1, 32, 8, nqb, nkb, seed=seed + 1,
                                 past_blocks=(kv_len - chunk) // SPARSE_BLOCK)


WORKLOADS = {
    "tiny": tiny,
    "decode": decode,
    "prefill": prefill,
    "mixed": mixed,
    "sparse": sparse,
}


E4M3_NAN_CODE = 0x7F


def with_kv8_pools(batch: Batch, *, seed: int, poison: bool = True, full_range: bool = False):
    """The batch with uint8 e4m3 code pools instead of bf16 ones, plus scales.

    Returns ``(batch8, k_scale [Hkv] fp32, v_scale [Hkv] fp32)``.  Context positions
    ``0 .. past-1`` of every sequence get random finite codes -- exponent fields 3..11, or,
    with ``full_range``, every finite code (zeros and subnormals included); all other slots
    get the NaN code (or 0).  ``k_new``/``v_new`` stay bf16 (they are quantised by the step
    itself).
    """
    g = torch.Generator().manual_seed(int(seed))
    fill = E4M3_NAN_CODE if poison else 0
    kp = torch.full(batch.k_pool.shape, fill, dtype=torch.uint8)
    vp = torch.full(batch.v_pool.shape, fill, dtype=torch.uint8)
    Hkv, D, P = batch.num_kv_heads, batch.head_dim, batch.page_size

    def draw(n):
        sign = torch.randint(0, 2, (n, Hkv, D), generator=g, dtype=torch.int32)
        lo, hi = (0, 16) if full_range else (3, 12)
        expo = torch.randint(lo, hi, (n, Hkv, D), generator=g, dtype=torch.int32)
        mant = torch.randint(0, 8, (n, Hkv, D), generator=g, dtype=torch.int32)
        code = (sign << 7) | (expo << 3) | mant
        code = torch.where((code & 0x7F) == 0x7F, code - 1, code)  # NaN -> largest finite
        return code.to(torch.uint8)

    bt = batch.block_table.to(torch.int64)
    for b, (kv, ql) in enumerate(zip(batch.kv_lens(), batch.q_lens())):
        past = kv - ql
        if past <= 0:
            continue
        kc, vc = draw(past), draw(past)
        pos = torch.arange(past)
        sl = pos % P
        if batch.layout == SEQ_MAJOR:
            pg = bt[b][pos // P]
            kp[pg, sl] = kc
            vp[pg, sl] = vc
        else:
            for h in range(Hkv):
                pg = bt[b, h][pos // P]
                kp[pg, sl] = kc[:, h]
                vp[pg, sl] = vc[:, h]
    k_scale = (0.005 + 0.015 * torch.rand(Hkv, generator=g)).to(torch.float32)
    v_scale = (0.05 + 0.15 * torch.rand(Hkv, generator=g)).to(torch.float32)
    out = dataclasses.replace(batch, k_pool=kp, v_pool=vp, k_logical=None, v_logical=None,
                              name=(batch.name + "-kv8") if batch.name else "kv8")
    return out, k_scale, v_scale
