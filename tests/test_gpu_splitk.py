"""pa_decode_splitk on the page-stream kernel (and pa_reduce after it) against
the fp64 oracle's per-partition partials.

Every partition row is compared element by element, the empty ones past
each context included (max -inf, sum 0, output 0, exactly); the maxima to
1e-4 absolute (scores are exact products of stored values, accumulated in
fp32), the normalisers to 1e-4 relative.  A normalised partial output is
an attention output over the partition's tokens, so it is held to the
decode tolerances of its dtype (fp32: 1e-5 max-abs; bf16 and FP8 pages:
2e-2 max-abs and 1e-2 mean-abs, the softmax weights going through bf16 or
fp16 tensor-core tiles), as is pa_reduce's output.  Unused cache slots hold
NaN, so an over-read shows.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_334_b200 import pa
from paged_kv_cache_334_b200 import workloads as wl

from _pa_helpers import assert_close, oracle_after_write, to_f64, upload

pytestmark = pytest.mark.gpu


def _splitk(d, P, maxp, B, Hq, D, err=None, sc=None):
    pm = torch.full((B, Hq, maxp), float("nan"), device="cuda")
    ps = torch.full_like(pm, float("nan"))
    po = torch.full((B, Hq, maxp, D), float("nan"), device="cuda")
    pa.pa_decode_splitk(d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                        d["context_lens"], P, pm, ps, po, err_word=err, **(sc or {}))
    return pm, ps, po


def _check_partials(got, ref, dtype, what):
    pm, ps, po = (to_f64(t) for t in got)
    rm, rs, ro = ref
    empty = rs == 0
    # empty partitions: exactly (-inf, 0, 0)
    assert np.all(np.isneginf(pm[empty])), f"{what}: empty partition max"
    assert np.all(ps[empty] == 0) and np.all(po[empty] == 0), f"{what}: empty partition"
    full = ~empty
    assert np.all(np.isfinite(pm[full])) and np.all(np.isfinite(po[full])), f"{what}: non-finite"
    np.testing.assert_allclose(pm[full], rm[full], rtol=0, atol=1e-4, err_msg=what)
    np.testing.assert_allclose(ps[full], rs[full], rtol=1e-4, atol=0, err_msg=what)
    assert_close(po[full], ro[full], dtype, what)


def _oracle_partials(w, P, maxp):
    kc, vc = w.key_cache.copy(), w.value_cache.copy()
    if w.slot_mapping is not None:
        assert oracle.write_kv_cache(kc, vc, w.k_new, w.v_new, w.slot_mapping) == 0
    rm, rs, ro, f = oracle.partials(w.q, kc, vc, w.block_tables, w.context_lens, P, maxp)
    return (rm, rs, ro), f


@pytest.mark.parametrize("P", [512, 256, 48])
def test_splitk_gqa_every_partition(P):
    """gqa_bf16 at full size: 512- and 256-token partitions, and 48 (three
    pages, not a power of two); two spare partitions per row stay empty."""
    w = wl.make_workload("gqa_bf16", seed=0)
    d = upload(w)
    pa.pa_write_kv_cache(d["key_cache"], d["value_cache"], d["k_new"], d["v_new"],
                         d["slot_mapping"])
    B, Hq, D = w.batch, w.num_q_heads, w.head_dim
    maxp = -(-w.max_blocks * w.block_size // P) + 2
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = _splitk(d, P, maxp, B, Hq, D, err)
    out = torch.empty_like(d["q"])
    pa.pa_reduce(out, *got, d["context_lens"], P, err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref, f = _oracle_partials(w, P, maxp)
    assert f == 0
    _check_partials(got, ref, w.dtype, f"gqa_bf16 P={P}")
    dec, _, _, _ = oracle_after_write(w)
    assert_close(to_f64(out), dec, w.dtype, f"gqa_bf16 split-K P={P} reduced")


def test_splitk_ragged_lengths_and_empty_sequences():
    """Lengths around page and partition edges, empty sequences, one long
    one; the CTA ranges end on partition boundaries whatever the mix."""
    ctx = [0, 1, 15, 16, 17, 511, 512, 513, 1023, 1024, 1025, 0, 7000, 33, 2047, 4096, 129, 5]
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=len(ctx), num_q_heads=32, num_kv_heads=8,
                           head_dim=128, block_size=16, context_lens=ctx, seed=21)
    d = upload(w)
    B, Hq, D, P = w.batch, w.num_q_heads, w.head_dim, 512
    maxp = -(-w.max_blocks * w.block_size // P)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = _splitk(d, P, maxp, B, Hq, D, err)
    out = torch.empty_like(d["q"])
    pa.pa_reduce(out, *got, d["context_lens"], P, err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref, f = _oracle_partials(w, P, maxp)
    assert f == 0
    _check_partials(got, ref, w.dtype, "ragged")
    dec, _, _, _ = oracle_after_write(w)
    assert_close(to_f64(out), dec, w.dtype, "ragged split-K reduced")


def test_splitk_many_sequences_multi_pass_prologue():
    """More sequences than threads per CTA (the prologue's scan runs in
    passes) and more than the cached length window; 32-token partitions."""
    rng = np.random.default_rng(5)
    ctx = rng.integers(0, 200, size=400).astype(np.int32)
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=400, num_q_heads=16, num_kv_heads=4,
                           head_dim=64, block_size=16, context_lens=ctx, seed=22)
    d = upload(w)
    B, Hq, D, P = w.batch, w.num_q_heads, w.head_dim, 32
    maxp = -(-w.max_blocks * w.block_size // P)
    got = _splitk(d, P, maxp, B, Hq, D)
    torch.cuda.synchronize()
    ref, f = _oracle_partials(w, P, maxp)
    assert f == 0
    _check_partials(got, ref, w.dtype, "400 sequences")


@pytest.mark.parametrize("hkv,hq,D,bs", [(4, 8, 64, 8), (8, 8, 128, 16), (4, 32, 128, 4)])
def test_splitk_fp32_pages(hkv, hq, D, bs):
    """fp32 pages on the page-stream kernel's CUDA-core consumers."""
    ctx = [300, 1, 0, 64, 257, 1000, 96]
    w = wl.custom_workload(dtype=wl.DTYPE_F32, batch=len(ctx), num_q_heads=hq,
                           num_kv_heads=hkv, head_dim=D, block_size=bs, context_lens=ctx,
                           seed=23)
    d = upload(w)
    B, P = w.batch, 64
    maxp = -(-w.max_blocks * w.block_size // P) + 1
    got = _splitk(d, P, maxp, B, hq, D)
    out = torch.empty_like(d["q"])
    pa.pa_reduce(out, *got, d["context_lens"], P)
    torch.cuda.synchronize()
    ref, f = _oracle_partials(w, P, maxp)
    assert f == 0
    _check_partials(got, ref, w.dtype, f"fp32 Hkv={hkv} Hq={hq} D={D} bs={bs}")
    dec, _, _, _ = oracle_after_write(w)
    assert_close(to_f64(out), dec, w.dtype, "fp32 split-K reduced")


def test_splitk_fp8_pages():
    """FP8 (E4M3) pages: partials against the oracle on the values the codes
    stand for (code * scale, exact in float64)."""
    w = wl.make_workload("gqa_fp8", seed=0)
    kc, vc = w.key_cache.copy(), w.value_cache.copy()
    assert oracle.write_kv_cache_fp8(kc, vc, w.k_new, w.v_new, w.slot_mapping, w.k_scale,
                                     w.v_scale) == 0

    def up(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        t = t.view(torch.float8_e4m3fn) if a.dtype == np.uint8 else t.view(torch.bfloat16)
        return t.cuda()

    d = dict(q=up(w.q), key_cache=up(kc), value_cache=up(vc),
             block_tables=torch.from_numpy(w.block_tables).cuda(),
             context_lens=torch.from_numpy(w.context_lens).cuda())
    sc = dict(k_scale=w.k_scale, v_scale=w.v_scale)
    B, Hq, D, P = w.batch, w.num_q_heads, w.head_dim, 512
    maxp = -(-w.max_blocks * w.block_size // P)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = _splitk(d, P, maxp, B, Hq, D, err, sc)
    out = torch.empty_like(d["q"])
    pa.pa_reduce(out, *got, d["context_lens"], P, err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rm, rs, ro, f = oracle.partials(oracle.widen(w.q), oracle.dequantize(kc, w.k_scale),
                                    oracle.dequantize(vc, w.v_scale), w.block_tables,
                                    w.context_lens, P, maxp)
    assert f == 0
    _check_partials(got, (rm, rs, ro), wl.DTYPE_BF16, "gqa_fp8")
    ref, _ = oracle.decode_fp8(w.q, kc, vc, w.k_scale, w.v_scale, w.block_tables,
                               w.context_lens, 1.0 / math.sqrt(w.head_dim))
    assert_close(to_f64(out), ref, wl.DTYPE_BF16, "gqa_fp8 split-K reduced")


def test_splitk_fp8_two_block_pages_at_four_kv_heads():
    """FP8 pages of 16-token blocks (two to a 32-token page) at 4 KV heads
    and 64-token partitions: partials and the reduced output against the
    oracle on the code values."""
    ctx = [1, 31, 33, 64, 65, 500, 1000]
    w = wl.custom_workload(dtype=wl.DTYPE_FP8, batch=len(ctx), num_q_heads=16,
                           num_kv_heads=4, head_dim=128, block_size=16, context_lens=ctx,
                           seed=24, k_scale=0.125, v_scale=0.75)

    def up(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        t = t.view(torch.float8_e4m3fn) if a.dtype == np.uint8 else t.view(torch.bfloat16)
        return t.cuda()

    d = dict(q=up(w.q), key_cache=up(w.key_cache), value_cache=up(w.value_cache),
             block_tables=torch.from_numpy(w.block_tables).cuda(),
             context_lens=torch.from_numpy(w.context_lens).cuda())
    sc = dict(k_scale=w.k_scale, v_scale=w.v_scale)
    B, Hq, D, P = w.batch, w.num_q_heads, w.head_dim, 64
    maxp = -(-w.max_blocks * w.block_size // P)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = _splitk(d, P, maxp, B, Hq, D, err, sc)
    out = torch.empty_like(d["q"])
    pa.pa_reduce(out, *got, d["context_lens"], P, err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rm, rs, ro, f = oracle.partials(oracle.widen(w.q), oracle.dequantize(w.key_cache, w.k_scale),
                                    oracle.dequantize(w.value_cache, w.v_scale), w.block_tables,
                                    w.context_lens, P, maxp)
    assert f == 0
    _check_partials(got, (rm, rs, ro), wl.DTYPE_BF16, "fp8 Hkv 4")
    ref, _ = oracle.decode_fp8(w.q, w.key_cache, w.value_cache, w.k_scale, w.v_scale,
                               w.block_tables, w.context_lens, 1.0 / math.sqrt(w.head_dim))
    assert_close(to_f64(out), ref, wl.DTYPE_BF16, "fp8 Hkv 4 split-K reduced")


def test_splitk_bad_metadata_on_the_stream_kernel():
    """A bad block id gives that partition sum -1 (the others are intact); a
    bad length gives empty partitions everywhere; both flagged."""
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=4, num_q_heads=32, num_kv_heads=8,
                           head_dim=128, block_size=16, context_lens=[40, 600, 300, 33],
                           seed=9, max_blocks=40)
    bt = w.block_tables.copy()
    cl = w.context_lens.copy()
    bt[0, 1] = w.num_blocks + 5       # tokens 16..31: partition 0 of sequence 0
    bt[1, 30] = -7                    # tokens 480..495: partition 1 (256-token partitions)
    cl[2] = 40 * 16 + 1               # longer than the table allows
    d = upload(w)
    d["block_tables"] = torch.from_numpy(bt).cuda()
    d["context_lens"] = torch.from_numpy(cl).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    P = 256
    maxp = -(-40 * 16 // P)
    pm, ps, po = _splitk(d, P, maxp, 4, 32, 128, err)
    torch.cuda.synchronize()
    assert int(err.item()) == pa.PA_DEVERR_BLOCK_ID | pa.PA_DEVERR_CONTEXT_LEN
    rm, rs, ro, flags = oracle.partials(w.q, w.key_cache, w.value_cache, bt, cl, P, maxp)
    assert flags != 0
    gs = to_f64(ps)
    assert np.all(gs[0, :, 0] == -1) and np.all(gs[1, :, 1] == -1)
    assert np.all(gs[2] == 0) and np.all(np.isneginf(to_f64(pm)[2]))
    assert np.all(to_f64(po)[2] == 0)
    # the untouched partitions match the oracle
    ok = rs > 0
    assert_close(to_f64(po)[ok], ro[ok], w.dtype, "intact partitions")
    np.testing.assert_allclose(gs[ok], rs[ok], rtol=1e-4, atol=0)


def test_splitk_one_partition_per_sequence_equals_decode():
    """Partitions longer than every context: one partition per sequence,
    which pa_reduce turns into pa_decode's result (up to rounding)."""
    w = wl.make_workload("gqa_bf16", seed=3)
    d = upload(w)
    pa.pa_write_kv_cache(d["key_cache"], d["value_cache"], d["k_new"], d["v_new"],
                         d["slot_mapping"])
    B, Hq, D = w.batch, w.num_q_heads, w.head_dim
    P = w.max_blocks * w.block_size
    got = _splitk(d, P, 1, B, Hq, D)
    out = torch.empty_like(d["q"])
    pa.pa_reduce(out, *got, d["context_lens"], P)
    dec = torch.empty_like(d["q"])
    pa.pa_decode(dec, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                 d["context_lens"])
    torch.cuda.synchronize()
    np.testing.assert_allclose(to_f64(out), to_f64(dec), rtol=0, atol=1e-2)
    ref, _, _, _ = oracle_after_write(w)
    assert_close(to_f64(out), ref, w.dtype, "one partition")
