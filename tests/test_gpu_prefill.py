"""pa_prefill (paged chunked prefill with the causal mask on tcgen05 tiles)
against the fp64 oracle's prefill of the same inputs: whole prompts and later
chunks of ragged lengths across the 128-row and 128-token tiles, every GQA
group width the kernel serves, head_dim 64 and 128, pages of 8 to 128
tokens, NaN in every slot past a context, sampled rows of 2048-token
prompts, and each flagged case.

Tolerance: bf16, <= 2e-2 max-abs and <= 1e-2 mean-abs (as for pa_decode).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_334_b200 import pa
from paged_kv_cache_334_b200 import workloads as wl

from _pa_helpers import assert_close, to_dev, to_f64, upload

pytestmark = pytest.mark.gpu


def _case(Hq, Hkv, D, bs, ctx, n, seed, max_blocks=None):
    """Sequences with context_lens ctx whose last n[b] tokens are the chunk."""
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=len(ctx), num_q_heads=Hq,
                           num_kv_heads=Hkv, head_dim=D, block_size=bs, context_lens=ctx,
                           seed=seed, max_blocks=max_blocks)
    rng = np.random.Generator(np.random.PCG64(seed + 7))
    T = int(sum(n))
    q = wl.to_storage(rng.standard_normal((max(T, 1), Hq, D), dtype=np.float32), wl.DTYPE_BF16)
    q = q[:T]
    qs = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    return w, q, qs


def _run(w, q, qs, err=None, cl=None, bt=None, mql=None):
    d = upload(w)
    qd = to_dev(q, wl.DTYPE_BF16)
    out = torch.full_like(qd, float("nan"))
    pa.pa_prefill(out, qd, d["key_cache"], d["value_cache"],
                  d["block_tables"] if bt is None else torch.from_numpy(bt).cuda(),
                  d["context_lens"] if cl is None else torch.from_numpy(cl).cuda(),
                  torch.from_numpy(qs).cuda(), max_query_len=mql, err_word=err)
    torch.cuda.synchronize()
    return to_f64(out)


SHAPES = [
    # Hq, Hkv, D, bs
    (32, 8, 128, 16),    # 4 heads per KV head: 32 tokens per tile
    (8, 8, 64, 16),      # 1 head per KV head: 128 tokens per tile, head_dim 64
    (64, 1, 128, 32),    # 64 heads per KV head: 2 tokens per tile
    (128, 1, 128, 64),   # 128 heads per KV head: 1 token per tile
    (16, 2, 128, 8),     # 8 heads per KV head, 8-token pages
    (32, 4, 64, 128),    # one page per K/V tile
]


@pytest.mark.parametrize("Hq,Hkv,D,bs", SHAPES)
def test_prompt_prefill(Hq, Hkv, D, bs):
    """Whole prompts (history == chunk) of ragged lengths around the tiles."""
    n = [1, 127, 128, 129, 300, 17] if Hq // Hkv <= 8 else [1, 5, 130, 64]
    w, q, qs = _case(Hq, Hkv, D, bs, n, n, seed=Hq + D + bs)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = _run(w, q, qs, err)
    assert int(err.item()) == 0
    ref, fl = oracle.prefill(q, w.key_cache, w.value_cache, w.block_tables, w.context_lens, qs)
    assert not fl.any()
    assert_close(got, ref, wl.DTYPE_BF16, f"prefill {Hq}/{Hkv} D{D} bs{bs}")


@pytest.mark.parametrize("Hq,Hkv,D,bs", SHAPES[:3])
def test_chunked_prefill(Hq, Hkv, D, bs):
    """Later chunks: histories longer than the chunk (NaN past each context)."""
    ctx = [500, 129, 1000, 64, 300]
    n = [37, 129, 200, 1, 0]
    w, q, qs = _case(Hq, Hkv, D, bs, ctx, n, seed=3 * Hq + bs)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = _run(w, q, qs, err)
    assert int(err.item()) == 0
    ref, _ = oracle.prefill(q, w.key_cache, w.value_cache, w.block_tables, w.context_lens, qs)
    assert_close(got, ref, wl.DTYPE_BF16, "chunked prefill")


def test_prefill_long_sampled():
    """4 prompts of 2048 tokens (32 query heads on 8 KV heads): sampled rows
    against the oracle's decode of the prefix ending at that token."""
    Hq, Hkv, D, bs = 32, 8, 128, 16
    n = [2048, 1500, 2048, 333]
    w, q, qs = _case(Hq, Hkv, D, bs, n, n, seed=11)
    got = _run(w, q, qs)
    rng = np.random.default_rng(0)
    for b in range(len(n)):
        for j in sorted(set(rng.integers(0, n[b], 12).tolist() + [0, n[b] - 1])):
            cl = np.array([j + 1], dtype=np.int32)
            ref, _ = oracle.decode(q[qs[b] + j][None], w.key_cache, w.value_cache,
                                   w.block_tables[b:b + 1], cl, 1.0 / math.sqrt(D))
            assert np.abs(got[qs[b] + j] - ref[0]).max() <= 2e-2, (b, j)


def test_prefill_flags_and_zeros():
    Hq, Hkv, D, bs = 32, 8, 128, 16
    ctx = [300, 200, 150]
    n = [300, 200, 150]
    w, q, qs = _case(Hq, Hkv, D, bs, ctx, n, seed=5)
    # sequence 1: more new tokens than its history holds
    cl = w.context_lens.copy()
    cl[1] = 100
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = _run(w, q, qs, err, cl=cl)
    assert int(err.item()) == oracle.FLAG_CONTEXT_LEN
    ref, fl = oracle.prefill(q, w.key_cache, w.value_cache, w.block_tables, cl, qs)
    assert fl.tolist() == [0, oracle.FLAG_CONTEXT_LEN, 0]
    assert_close(got, ref, wl.DTYPE_BF16, "flagged length")
    # sequence 2: a block id past the pool
    bt = w.block_tables.copy()
    bt[2, 3] = w.num_blocks + 5
    err.zero_()
    got = _run(w, q, qs, err, bt=bt)
    assert int(err.item()) == oracle.FLAG_BLOCK_ID
    ref, _ = oracle.prefill(q, w.key_cache, w.value_cache, bt, w.context_lens, qs)
    assert_close(got, ref, wl.DTYPE_BF16, "flagged block")
    # a query_start past num_tokens: that sequence's rows are not written
    qs2 = qs.copy()
    qs2[3] = qs2[3] + 1
    err.zero_()
    got = _run(w, q, qs2, err)
    assert int(err.item()) & oracle.FLAG_CONTEXT_LEN
    assert np.isnan(got[qs[2]:]).all()
    # a chunk longer than max_query_len: flagged, the covered rows zeroed
    err.zero_()
    got = _run(w, q, qs, err, mql=128)
    assert int(err.item()) == oracle.FLAG_CONTEXT_LEN
    assert not got[:128].any()
