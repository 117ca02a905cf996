"""Seeded synthetic workloads for paged decode attention.

This module only draws inputs: random values, context lengths, a shuffled
pool of physical blocks and the block tables that a simple allocator hands
out.  It holds none of the attention arithmetic and imports neither the CUDA
binding nor the oracle, so both sides can be fed the same arrays.

The allocator here plays the Block Manager of the pages (page "Implementing
teaching PagedAttention: reading the historical KV cache from the block
table", opening section: free blocks are handed out for prefill and a slot
is appended for each decode step).  It records where it put every token; the
slot of a sequence's newest token is reported as the flat integer
``physical_block_id * block_size + block_offset`` of the place it reserved.

Workload recipes (all values N(0, 1); bf16 values are drawn in fp32 and
rounded to nearest-even by torch's cast; every array is host memory):

``tiny_fp32``
    batch 3, 4 query / 4 KV heads, head_dim 64, block_size 4, 16 blocks,
    context_lens [5, 9, 12]; sequence 0's table is fixed to [7, 2, 9], the
    other tables are drawn without replacement from the remaining blocks.
``gqa_bf16``
    batch 32, 32 / 8 heads, head_dim 128, block_size 16, context lengths
    uniform in [128, 2048], blocks a seeded permutation of a pool with 20 %
    slack.
``mixed_bf16``
    batch 128, 32 / 8 heads, head_dim 128, block_size 16, lengths drawn from
    {128: 50 %, 4096: 35 %, 16000: 15 %} plus uniform jitter in [0, 15],
    scattered tables from a 20 %-slack pool.
``long_bf16``
    batch 4, context 131072 each, 32 / 8 heads, head_dim 128,
    block_size 16, a seeded permutation of exactly the blocks needed,
    512-token partitions.
``mqa_prefix_bf16``
    batch 256, 64 query heads / 1 KV head, head_dim 128, block_size 32;
    every table starts with the same 64 shared prefix blocks (2048 tokens)
    followed by a private suffix of uniform [1, 1024] tokens in scattered
    blocks (20 % slack).

``gqa_fp8``
    gqa_bf16's shape and lengths with FP8 pages: caches of E4M3 codes
    (uint8) standing for code * 0.25 (K) and code * 0.5 (V), the codes drawn
    directly (sign, exponent field 3..9, mantissa uniform), NaN code 0x7F
    in unused slots; q and the new rows in bf16.

In every workload but ``tiny_fp32`` the last token of each sequence is the
token of the current decode step: its K/V rows are returned in
``k_new``/``v_new`` with the slot reserved for it in ``slot_mapping``, and
its place in the cache is filled with NaN until the cache write runs.  Slots
of unreferenced blocks and slots past each context length are NaN too, so a
kernel that reads outside the visible history produces NaN.

Prefill inputs (``prefill_workload``) reuse a bf16 workload's pool, tables
and lengths with the held-back newest tokens put into their slots, and draw
a fresh q (N(0, 1), bf16) with one row per chunk token: whole prompts, or
the last tokens of each context as the chunk of a chunked prefill.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

DTYPE_F32 = "f32"
DTYPE_BF16 = "bf16"
DTYPE_FP8 = "fp8_e4m3"
FP8_K_SCALE = 0.25  # the fp8 workloads' per-tensor scales
FP8_V_SCALE = 0.5

WORKLOADS = ("tiny_fp32", "gqa_bf16", "mixed_bf16", "long_bf16", "mqa_prefix_bf16", "gqa_fp8")

_BF16_NAN = np.uint16(0x7FC0)


@dataclasses.dataclass
class Workload:
    name: str
    # "f32" (float32 arrays), "bf16" (uint16 arrays of bf16 bits) or
    # "fp8_e4m3": caches of E4M3 codes (uint8) standing for code * k_scale /
    # code * v_scale, with q and the new rows in bf16
    dtype: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    max_blocks: int
    q: np.ndarray  # [B, Hq, D]
    key_cache: np.ndarray  # [NB, bs, Hkv, D]
    value_cache: np.ndarray  # [NB, bs, Hkv, D]
    block_tables: np.ndarray  # [B, MB] int32, unused entries -1
    context_lens: np.ndarray  # [B] int32
    k_new: Optional[np.ndarray] = None  # [N, Hkv, D]
    v_new: Optional[np.ndarray] = None
    slot_mapping: Optional[np.ndarray] = None  # [N] int64
    partition_tokens: Optional[int] = None
    seed: int = 0
    description: str = ""
    shared_prefix_blocks: int = 0  # leading table entries every sequence shares
    k_scale: float = 1.0  # fp8_e4m3 caches: value = code * scale
    v_scale: float = 1.0

    @property
    def elem_bytes(self) -> int:
        """Bytes of one cache element."""
        return 4 if self.dtype == DTYPE_F32 else 1 if self.dtype == DTYPE_FP8 else 2

    @property
    def act_bytes(self) -> int:
        """Bytes of one element of q, out and the new rows."""
        return 4 if self.dtype == DTYPE_F32 else 2

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads


def to_storage(values_f32: np.ndarray, dtype: str) -> np.ndarray:
    """fp32 values -> storage array: float32 as is, bf16 as uint16 bits (RNE)."""
    if dtype == DTYPE_F32:
        return np.ascontiguousarray(values_f32, dtype=np.float32)
    import torch

    t = torch.from_numpy(np.ascontiguousarray(values_f32, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.uint16).numpy().copy()


def _nan_value(dtype: str):
    return np.float32("nan") if dtype == DTYPE_F32 else _BF16_NAN


def _normal_storage(rng: np.random.Generator, shape, dtype: str,
                    chunk: int = 1 << 26) -> np.ndarray:
    """N(0,1) draws in storage format, generated in chunks to bound memory."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32 if dtype == DTYPE_F32 else np.uint16)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        out[s:e] = to_storage(rng.standard_normal(e - s, dtype=np.float32), dtype)
    return out.reshape(shape)


def _pages(ctx: int, bs: int) -> int:
    return (ctx + bs - 1) // bs


def _e4m3_codes(rng: np.random.Generator, shape, chunk: int = 1 << 26) -> np.ndarray:
    """Random E4M3 codes (uint8): sign, exponent field 3..9 (magnitudes
    2^-4 .. 1.875 * 2^2) and mantissa drawn uniformly; no value is computed."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint8)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        sign = rng.integers(0, 2, size=e - s, dtype=np.uint8) << 7
        expo = rng.integers(3, 10, size=e - s, dtype=np.uint8) << 3
        mant = rng.integers(0, 8, size=e - s, dtype=np.uint8)
        out[s:e] = sign | expo | mant
    return out.reshape(shape)


_E4M3_NAN = np.uint8(0x7F)


def _finish(name, dtype, rng, B, Hq, Hkv, D, bs, NB, MB, ctx, tables,
            new_tokens: bool, partition_tokens=None, seed=0, description=""):
    """Draw q and cache contents, poison unused slots, peel off new tokens."""
    fp8 = dtype == DTYPE_FP8
    q = _normal_storage(rng, (B, Hq, D), DTYPE_BF16 if fp8 else dtype)
    if fp8:
        kc = _e4m3_codes(rng, (NB, bs, Hkv, D))
        vc = _e4m3_codes(rng, (NB, bs, Hkv, D))
        nan = _E4M3_NAN
    else:
        kc = _normal_storage(rng, (NB, bs, Hkv, D), dtype)
        vc = _normal_storage(rng, (NB, bs, Hkv, D), dtype)
        nan = _nan_value(dtype)
    # Slots that hold a visible token of some sequence.
    live = np.zeros((NB, bs), dtype=bool)
    for b in range(B):
        for lb in range(_pages(int(ctx[b]), bs)):
            n_valid = min(bs, int(ctx[b]) - lb * bs)
            live[tables[b, lb], :n_valid] = True
    kc[~live] = nan
    vc[~live] = nan
    k_new = v_new = slots = None
    if new_tokens:
        rows = [b for b in range(B) if ctx[b] > 0]
        if fp8:
            # the new rows arrive in bf16; the write quantises them
            k_new = _normal_storage(rng, (len(rows), Hkv, D), DTYPE_BF16)
            v_new = _normal_storage(rng, (len(rows), Hkv, D), DTYPE_BF16)
        else:
            k_new = np.empty((len(rows), Hkv, D), dtype=kc.dtype)
            v_new = np.empty_like(k_new)
        slots = np.empty(len(rows), dtype=np.int64)
        for i, b in enumerate(rows):
            t = int(ctx[b]) - 1
            pb, off = int(tables[b, t // bs]), t % bs  # where the allocator put it
            if not fp8:
                k_new[i] = kc[pb, off]
                v_new[i] = vc[pb, off]
            kc[pb, off] = nan
            vc[pb, off] = nan
            slots[i] = pb * bs + off
    return Workload(name=name, dtype=dtype, batch=B, num_q_heads=Hq,
                    num_kv_heads=Hkv, head_dim=D, block_size=bs, num_blocks=NB,
                    max_blocks=MB, q=q, key_cache=kc, value_cache=vc,
                    block_tables=tables, context_lens=ctx.astype(np.int32),
                    k_new=k_new, v_new=v_new, slot_mapping=slots,
                    partition_tokens=partition_tokens, seed=seed,
                    description=description)


def _scattered_tables(rng, ctx, bs, MB, slack=0.2, prefix_blocks=0):
    """Tables from a seeded permutation of a pool with `slack` spare blocks.

    With prefix_blocks > 0 every table starts with the same prefix blocks
    (the first ones of the permutation); suffix pages follow."""
    B = len(ctx)
    need = [_pages(int(c), bs) - prefix_blocks for c in ctx]
    total = prefix_blocks + sum(need)
    NB = int(math.ceil((1.0 + slack) * total))
    perm = rng.permutation(NB).astype(np.int32)
    tables = np.full((B, MB), -1, dtype=np.int32)
    prefix = perm[:prefix_blocks]
    pos = prefix_blocks
    for b in range(B):
        tables[b, :prefix_blocks] = prefix
        tables[b, prefix_blocks:prefix_blocks + need[b]] = perm[pos:pos + need[b]]
        pos += need[b]
    return tables, NB


def make_workload(name: str, seed: int = 0, batch: Optional[int] = None,
                  block_size: Optional[int] = None) -> Workload:
    """Build one of the named workloads.  `batch` overrides the batch size
    (used for reduced-size variants of the large workloads); `block_size`
    (a power of two) overrides the page size of gqa_bf16, mixed_bf16 and
    long_bf16 (the same lengths and values, paged differently: a page-size
    sweep)."""
    if block_size is not None:
        if name not in ("gqa_bf16", "mixed_bf16", "long_bf16", "gqa_fp8"):
            raise ValueError("block_size override is for gqa_bf16, mixed_bf16, long_bf16, "
                             f"gqa_fp8, not {name}")
        if block_size < 1 or block_size & (block_size - 1):
            raise ValueError(f"block_size must be a power of two, not {block_size}")
    rng = np.random.Generator(np.random.PCG64(seed))
    if name == "tiny_fp32":
        B, Hq, Hkv, D, bs, NB = 3, 4, 4, 64, 4, 16
        ctx = np.array([5, 9, 12], dtype=np.int32)
        MB = 3
        tables = np.full((B, MB), -1, dtype=np.int32)
        tables[0] = [7, 2, 9]
        rest = np.array([x for x in range(NB) if x not in (7, 2, 9)], dtype=np.int32)
        drawn = rng.choice(rest, size=_pages(9, bs) + _pages(12, bs), replace=False)
        tables[1] = drawn[:3]
        tables[2] = drawn[3:6]
        return _finish(name, DTYPE_F32, rng, B, Hq, Hkv, D, bs, NB, MB, ctx,
                       tables, new_tokens=False, seed=seed,
                       description="B3 Hq4/Hkv4 D64 bs4 NB16 ctx[5,9,12] fp32")
    if name == "gqa_bf16":
        B = batch or 32
        Hq, Hkv, D, bs = 32, 8, 128, block_size or 16
        ctx = rng.integers(128, 2048, size=B, endpoint=True).astype(np.int32)
        MB = _pages(2048, bs)
        tables, NB = _scattered_tables(rng, ctx, bs, MB)
        return _finish(name, DTYPE_BF16, rng, B, Hq, Hkv, D, bs, NB, MB, ctx,
                       tables, new_tokens=True, seed=seed,
                       description=f"B{B} Hq32/Hkv8 D128 bs{bs} ctx~U[128,2048] bf16")
    if name == "mixed_bf16":
        B = batch or 128
        Hq, Hkv, D, bs = 32, 8, 128, block_size or 16
        base = rng.choice(np.array([128, 4096, 16000]), size=B, p=[0.5, 0.35, 0.15])
        jitter = rng.integers(0, 15, size=B, endpoint=True)
        ctx = (base + jitter).astype(np.int32)
        MB = _pages(16000 + 15, bs)
        tables, NB = _scattered_tables(rng, ctx, bs, MB)
        return _finish(name, DTYPE_BF16, rng, B, Hq, Hkv, D, bs, NB, MB, ctx,
                       tables, new_tokens=True, seed=seed,
                       description=f"B{B} Hq32/Hkv8 D128 bs{bs} ctx {{128,4096,16000}}+U[0,15] bf16")
    if name == "long_bf16":
        B = batch or 4
        Hq, Hkv, D, bs, L = 32, 8, 128, block_size or 16, 131072
        ctx = np.full(B, L, dtype=np.int32)
        MB = _pages(L, bs)
        tables, NB = _scattered_tables(rng, ctx, bs, MB, slack=0.0)
        return _finish(name, DTYPE_BF16, rng, B, Hq, Hkv, D, bs, NB, MB, ctx,
                       tables, new_tokens=True, partition_tokens=512, seed=seed,
                       description=f"B{B} ctx131072 Hq32/Hkv8 D128 bs{bs} bf16, 512-token partitions")
    if name == "mqa_prefix_bf16":
        B = batch or 256
        Hq, Hkv, D, bs, prefix = 64, 1, 128, 32, 2048
        suffix = rng.integers(1, 1024, size=B, endpoint=True)
        ctx = (prefix + suffix).astype(np.int32)
        MB = _pages(prefix + 1024, bs)
        tables, NB = _scattered_tables(rng, ctx, bs, MB, prefix_blocks=prefix // bs)
        w = _finish(name, DTYPE_BF16, rng, B, Hq, Hkv, D, bs, NB, MB, ctx,
                    tables, new_tokens=True, seed=seed,
                    description=f"B{B} Hq64/Hkv1 D128 bs32, 2048 shared prefix + U[1,1024] suffix, bf16")
        w.shared_prefix_blocks = prefix // bs
        return w
    if name == "gqa_fp8":
        # gqa_bf16's shape and lengths with FP8 (E4M3) pages
        B = batch or 32
        Hq, Hkv, D, bs = 32, 8, 128, block_size or 16
        ctx = rng.integers(128, 2048, size=B, endpoint=True).astype(np.int32)
        MB = _pages(2048, bs)
        tables, NB = _scattered_tables(rng, ctx, bs, MB)
        w = _finish(name, DTYPE_FP8, rng, B, Hq, Hkv, D, bs, NB, MB, ctx, tables,
                    new_tokens=True, seed=seed,
                    description=f"B{B} Hq32/Hkv8 D128 bs{bs} ctx~U[128,2048] fp8_e4m3 pages")
        w.k_scale, w.v_scale = FP8_K_SCALE, FP8_V_SCALE
        return w
    raise ValueError(f"unknown workload {name!r}; known: {WORKLOADS}")


def custom_workload(*, dtype: str, batch: int, num_q_heads: int, num_kv_heads: int,
                    head_dim: int, block_size: int, context_lens, seed: int = 0,
                    slack: float = 0.2, max_blocks: Optional[int] = None,
                    new_tokens: bool = False, prefix_blocks: int = 0,
                    k_scale: float = FP8_K_SCALE, v_scale: float = FP8_V_SCALE) -> Workload:
    """A workload with explicit context lengths (edge cases, sweeps).  With
    prefix_blocks > 0 every table starts with the same physical blocks (a
    shared prompt prefix); every context must cover them.  k_scale / v_scale
    are the per-tensor scales of fp8_e4m3 caches."""
    rng = np.random.Generator(np.random.PCG64(seed))
    ctx = np.asarray(context_lens, dtype=np.int32)
    need = max([_pages(int(c), block_size) for c in ctx] + [1])
    MB = max_blocks if max_blocks is not None else need
    if prefix_blocks:
        assert all(int(c) >= prefix_blocks * block_size for c in ctx), "context shorter than prefix"
    tables, NB = _scattered_tables(rng, np.maximum(ctx, 0), block_size, MB, slack=slack,
                                   prefix_blocks=prefix_blocks)
    NB = max(NB, 1)
    w = _finish("custom", dtype, rng, batch, num_q_heads, num_kv_heads, head_dim,
                block_size, NB, MB, ctx, tables,
                new_tokens=new_tokens, seed=seed,
                description=f"custom ctx={list(map(int, ctx))[:8]}...")
    w.shared_prefix_blocks = prefix_blocks
    if dtype == DTYPE_FP8:
        w.k_scale, w.v_scale = k_scale, v_scale
    return w


def roofline_bytes(w: Workload, include_write: bool = True) -> int:
    """Algorithmic HBM bytes of one decode step: unique K/V bytes of the
    visible tokens (shared pages counted once), block tables, context
    lengths, q and out, plus the new-token rows and slots when written."""
    row = w.num_kv_heads * w.head_dim * w.elem_bytes
    seen = set()
    kv = 0
    for b in range(w.batch):
        ctx = int(w.context_lens[b])
        for lb in range(_pages(ctx, w.block_size)):
            pb = int(w.block_tables[b, lb])
            n_valid = min(w.block_size, ctx - lb * w.block_size)
            if pb in seen:
                continue
            seen.add(pb)
            kv += 2 * n_valid * row
    qo = 2 * w.batch * w.num_q_heads * w.head_dim * w.act_bytes
    meta = w.block_tables.size * 4 + w.context_lens.size * 4
    extra = 0
    if include_write and w.slot_mapping is not None:
        # new rows read once and stored once (as cache elements), K and V
        n_new = w.slot_mapping.size
        extra = (w.k_new.nbytes + w.v_new.nbytes + 2 * n_new * row +
                 w.slot_mapping.nbytes)
    return int(kv + qo + meta + extra)


# ---------------------------------------------------------------------------
# paged (chunked) prefill inputs
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class PrefillWorkload:
    """Prefill inputs over a decode workload's pool: sequence b's chunk is
    rows query_start[b] .. query_start[b+1]-1 of q, the last chunk_lens[b]
    tokens of its context_lens[b]-token history, every token of which is
    stored in the pool of `base`."""
    base: Workload          # pool, tables and lengths; no pending new tokens
    q: np.ndarray           # [T, Hq, D] bf16 storage
    query_start: np.ndarray  # [B + 1] int32
    chunk_lens: np.ndarray   # [B] int32
    description: str = ""

    @property
    def num_tokens(self) -> int:
        return int(self.query_start[-1])

    @property
    def max_query_len(self) -> int:
        return int(self.chunk_lens.max()) if self.chunk_lens.size else 0


def prefill_workload(w: Workload, chunk: Optional[int] = None, seed: int = 0) -> PrefillWorkload:
    """Prefill inputs over w's pool, tables and lengths: whole prompts (chunk
    None: each context is one prompt, as the teaching page's prefill stores a
    prompt's K/V and attends over it causally) or, with chunk = c, the last
    min(c, ctx) tokens of each context as the chunk of a chunked prefill.
    The newest tokens w held back for its decode step are put into their
    slots, so every context token is stored; q is drawn afresh (N(0, 1),
    rounded to bf16)."""
    if w.dtype != DTYPE_BF16:
        raise ValueError(f"prefill inputs are bf16, not {w.dtype}")
    kc, vc = w.key_cache.copy(), w.value_cache.copy()
    if w.slot_mapping is not None:
        bs = w.block_size
        for i, s in enumerate(w.slot_mapping.tolist()):
            kc[s // bs, s % bs] = w.k_new[i]
            vc[s // bs, s % bs] = w.v_new[i]
    ctx = w.context_lens.astype(np.int64)
    n = ctx if chunk is None else np.minimum(ctx, int(chunk))
    qs = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    rng = np.random.Generator(np.random.PCG64(seed + 0x5EED))
    q = _normal_storage(rng, (int(qs[-1]), w.num_q_heads, w.head_dim), DTYPE_BF16)
    base = dataclasses.replace(w, key_cache=kc, value_cache=vc, k_new=None, v_new=None,
                               slot_mapping=None)
    what = "whole prompts" if chunk is None else f"last <= {chunk} tokens of each context"
    return PrefillWorkload(base=base, q=q, query_start=qs, chunk_lens=n.astype(np.int32),
                           description=f"{w.name} pool, {what}, {int(qs[-1])} query tokens")


def prefill_flops(pw: PrefillWorkload) -> float:
    """QK and PV of every (chunk token, query head, visible position): chunk
    token j of a chunk of n at the end of a ctx-token history sees ctx - n +
    j + 1 positions, 2 * 2 * head_dim flops each."""
    w = pw.base
    ctx = w.context_lens.astype(np.float64)
    n = pw.chunk_lens.astype(np.float64)
    pairs = float(np.sum(n * (ctx - n) + n * (n + 1) / 2))
    return 4.0 * w.head_dim * w.num_q_heads * pairs


def prefill_roofline_bytes(pw: PrefillWorkload) -> int:
    """Algorithmic HBM bytes of one prefill call: unique K/V bytes of every
    context token, tables, lengths, query_start, and q and out of the chunk
    tokens (read and written once)."""
    w = pw.base
    decode_qo = 2 * w.batch * w.num_q_heads * w.head_dim * w.act_bytes
    qo = 2 * pw.num_tokens * w.num_q_heads * w.head_dim * w.act_bytes
    return int(roofline_bytes(w, include_write=False) - decode_qo + qo + pw.query_start.nbytes)
