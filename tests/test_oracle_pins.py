"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each test names the passage or the mathematical fact it rests on and is
chosen so that a plausible slip in the oracle (a dropped scale, a wrong sign
in the exponent, swapped division / modulo, a transposed operand, a wrong
GQA head index, a missing normalisation, reading past the context) fails at
least one of them.  Pages cited:

* "From correct to faster: the PagedAttention optimisation route"
  (yjxyzxyz.cn, article oHue8hrF) -- the optimisation-route page;
* "Implementing teaching PagedAttention: reading the historical KV cache from
  the block table" (yjxyzxyz.cn, article wVdUWYLj) -- the teaching page.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_334_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _paged_from_contiguous(k_contig, v_contig, table, bs, num_blocks, fill=np.nan):
    """Build a paged cache by cutting contiguous [ctx, Hkv, D] rows into
    whole pages and dropping page i at physical block table[i] (page-level
    reshape, not the per-token formula)."""
    ctx, Hkv, D = k_contig.shape
    n_pages = -(-ctx // bs)
    kc = np.full((num_blocks, bs, Hkv, D), fill, dtype=np.float32)
    vc = np.full_like(kc, fill)
    pad = n_pages * bs - ctx
    kp = np.concatenate([k_contig, np.full((pad, Hkv, D), fill, np.float32)]).reshape(n_pages, bs, Hkv, D)
    vp = np.concatenate([v_contig, np.full((pad, Hkv, D), fill, np.float32)]).reshape(n_pages, bs, Hkv, D)
    kc[np.asarray(table[:n_pages])] = kp
    vc[np.asarray(table[:n_pages])] = vp
    return kc, vc


# --------------------------------------------------------------------------
# Address mapping: the pages' worked examples (bit-exact)
# --------------------------------------------------------------------------

def test_worked_example_mapping_7_2_9():
    """Teaching page, "PagedAttention changes how the KV cache is accessed":
    block size 4, table [7, 2, 9], tokens 0..8 -> (block, offset)."""
    rows = _read_golden("worked_example_7_2_9.txt")
    bs = int([r for r in rows if r[0] == "block_size"][0][1])
    table = [int(x) for x in [r for r in rows if r[0] == "block_table"][0][1:]]
    maps = [tuple(map(int, r[1:])) for r in rows if r[0] == "map"]
    assert len(maps) == 9
    for t, pb_exp, off_exp in maps:
        pb, off, f = oracle.map_token(table, t, bs, num_blocks=16)
        assert f == 0
        assert (pb, off) == (pb_exp, off_exp), t


def test_worked_example_token5_reads_key_cache_2_1():
    """Teaching page, "First define a simple KV cache layout": logical token
    5 of table [7, 2, 9] is key_cache[2, 1] / value_cache[2, 1]."""
    rows = _read_golden("worked_example_7_2_9.txt")
    t, lb, off, pb = [int(x) for x in [r for r in rows if r[0] == "read"][0][1:]]
    bs, Hkv, D, NB = 4, 2, 8, 16
    kc = np.zeros((NB, bs, Hkv, D), np.float32)
    vc = np.zeros_like(kc)
    kc[pb, off] = 5.25
    vc[pb, off] = -3.5
    keys, vals, f = oracle.gather_kv(kc, vc, [7, 2, 9], context_len=6)
    assert f == 0
    assert np.all(keys[t] == 5.25) and np.all(vals[t] == -3.5)
    # every other gathered row comes from elsewhere (zeros here)
    others = [i for i in range(6) if i != t]
    assert np.all(keys[others] == 0.0) and np.all(vals[others] == 0.0)
    assert t // bs == lb and t % bs == off


def test_worked_example_slot_write_lands_where_token5_is_read():
    """Teaching page, "Writing slots and reading the block table must agree":
    the slot the allocator reserves for token 5 of table [7, 2, 9] is
    (block 2, offset 1), encoded 2*4+1 = 9; the byte copy lands at
    key_cache[2, 1] and nowhere else, and the gather reads it back."""
    bs, Hkv, D, NB = 4, 2, 8, 16
    rng = np.random.default_rng(3)
    kc = rng.standard_normal((NB, bs, Hkv, D)).astype(np.float32)
    vc = rng.standard_normal((NB, bs, Hkv, D)).astype(np.float32)
    k0, v0 = kc.copy(), vc.copy()
    kn = rng.standard_normal((1, Hkv, D)).astype(np.float32)
    vn = rng.standard_normal((1, Hkv, D)).astype(np.float32)
    assert oracle.write_kv_cache(kc, vc, kn, vn, np.array([2 * 4 + 1])) == 0
    assert kc[2, 1].tobytes() == kn[0].tobytes() and vc[2, 1].tobytes() == vn[0].tobytes()
    mask = np.ones((NB, bs), bool)
    mask[2, 1] = False
    assert np.array_equal(kc[mask], k0[mask]) and np.array_equal(vc[mask], v0[mask])
    keys, vals, f = oracle.gather_kv(kc, vc, [7, 2, 9], context_len=6)
    assert keys[5].tobytes() == kn[0].astype(np.float64).tobytes()


def test_batch_example_tables_cover_their_contexts():
    """Teaching page, "Extending to a batch": A [7,2,9] ctx 10, B [4,1]
    ctx 6, C [8,5,3,6] ctx 15.  Each table is exactly ceil(ctx/4) long:
    every visible token maps inside it, the last token into the last entry."""
    rows = _read_golden("batch_example_tables.txt")
    bs = int([r for r in rows if r[0] == "block_size"][0][1])
    seqs = [r for r in rows if r[0] == "seq"]
    assert [s[1] for s in seqs] == ["A", "B", "C"]
    for s in seqs:
        ctx = int(s[2])
        table = [int(x) for x in s[3:]]
        assert len(table) == -(-ctx // bs)
        seen = []
        for t in range(ctx):
            pb, off, f = oracle.map_token(table, t, bs, num_blocks=16)
            assert f == 0
            seen.append((pb, off))
        assert seen[-1][0] == table[-1]
        assert len(set(seen)) == ctx  # distinct slots for distinct tokens
        # one past the table's reach is flagged, not read
        _, _, f = oracle.map_token(table, len(table) * bs, bs, num_blocks=16)
        assert f == oracle.FLAG_CONTEXT_LEN


# --------------------------------------------------------------------------
# Paged attention == contiguous attention (teaching page, "Aligning with a
# contiguous KV cache"; optimisation-route page, "Guard correctness before
# writing the fast version")
# --------------------------------------------------------------------------

@pytest.mark.parametrize("ctx,bs", [(1, 4), (3, 4), (4, 4), (5, 4), (37, 8), (100, 16)])
def test_paged_equals_contiguous_bitwise(ctx, bs):
    rng = np.random.default_rng(ctx * 131 + bs)
    Hq, Hkv, D = 8, 2, 16
    k = rng.standard_normal((ctx, Hkv, D)).astype(np.float32)
    v = rng.standard_normal((ctx, Hkv, D)).astype(np.float32)
    q = rng.standard_normal((1, Hq, D)).astype(np.float32)
    n_pages = -(-ctx // bs)
    NB = n_pages + 5
    table = rng.permutation(NB)[:n_pages].astype(np.int32)
    kc, vc = _paged_from_contiguous(k, v, table, bs, NB)
    out_paged, flags = oracle.decode(q, kc, vc, table[None, :], np.array([ctx], np.int32))
    assert flags[0] == 0
    out_contig = oracle.attention(q[0].astype(np.float64), k.astype(np.float64),
                                  v.astype(np.float64), 1.0 / math.sqrt(D))
    assert np.array_equal(out_paged[0], out_contig)
    assert np.all(np.isfinite(out_paged))


# --------------------------------------------------------------------------
# Special case that reduces to a library routine: torch's scaled dot product
# attention in float64 (scale 1/sqrt(D), GQA by contiguous head groups)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("Hq,Hkv,D,ctx", [(4, 4, 64, 12), (32, 8, 128, 77), (16, 1, 32, 50), (6, 3, 8, 1)])
def test_matches_torch_sdpa_float64(Hq, Hkv, D, ctx):
    rng = np.random.default_rng(Hq * 7 + ctx)
    bs = 4
    k = rng.standard_normal((ctx, Hkv, D)).astype(np.float32)
    v = rng.standard_normal((ctx, Hkv, D)).astype(np.float32)
    q = rng.standard_normal((1, Hq, D)).astype(np.float32)
    n_pages = -(-ctx // bs)
    table = rng.permutation(n_pages + 3)[:n_pages].astype(np.int32)
    kc, vc = _paged_from_contiguous(k, v, table, bs, n_pages + 3)
    out, flags = oracle.decode(q, kc, vc, table[None, :], np.array([ctx], np.int32))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q.astype(np.float64)).reshape(1, Hq, 1, D),
        torch.from_numpy(k.astype(np.float64)).permute(1, 0, 2).reshape(1, Hkv, ctx, D),
        torch.from_numpy(v.astype(np.float64)).permute(1, 0, 2).reshape(1, Hkv, ctx, D),
        enable_gqa=True,
    ).reshape(Hq, D).numpy()
    np.testing.assert_allclose(out[0], ref, rtol=0, atol=1e-12)


def test_bf16_widening_matches_torch_conversion():
    rng = np.random.default_rng(0)
    bits = wl.to_storage(rng.standard_normal(4096).astype(np.float32) * 50, wl.DTYPE_BF16)
    bits = np.concatenate([bits, np.array([0x0000, 0x8000, 0x7F80, 0xFF80, 0x0001, 0x7F7F], np.uint16)])
    ref = torch.from_numpy(bits.copy()).view(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.widen(bits), ref)


# --------------------------------------------------------------------------
# Closed forms
# --------------------------------------------------------------------------

def _one_seq(k, v, q, bs=4, seed=0):
    ctx = k.shape[0]
    rng = np.random.default_rng(seed)
    n_pages = -(-ctx // bs)
    table = rng.permutation(n_pages + 2)[:n_pages].astype(np.int32)
    kc, vc = _paged_from_contiguous(k.astype(np.float32), v.astype(np.float32), table, bs, n_pages + 2)
    out, flags = oracle.decode(q.astype(np.float32)[None], kc, vc, table[None], np.array([ctx], np.int32))
    assert flags[0] == 0
    return out[0]


def test_context_len_one_returns_v0_exactly():
    rng = np.random.default_rng(1)
    k = rng.standard_normal((1, 2, 16))
    v = rng.standard_normal((1, 2, 16)).astype(np.float32)
    q = rng.standard_normal((4, 16))
    out = _one_seq(k, v, q)
    for hq in range(4):
        assert np.array_equal(out[hq], v[0, hq // 2].astype(np.float64))


def test_constant_keys_give_mean_of_values():
    rng = np.random.default_rng(2)
    ctx = 23
    k = np.tile(rng.standard_normal((1, 1, 32)), (ctx, 1, 1))
    v = rng.standard_normal((ctx, 1, 32)).astype(np.float32)
    q = rng.standard_normal((3, 32))
    out = _one_seq(k, v, q)
    np.testing.assert_allclose(out, np.tile(v.astype(np.float64).mean(axis=0), (3, 1)), atol=1e-13)


def test_constant_values_are_reproduced():
    rng = np.random.default_rng(3)
    ctx = 41
    k = rng.standard_normal((ctx, 1, 32))
    v = np.tile(rng.standard_normal((1, 1, 32)), (ctx, 1, 1)).astype(np.float32)
    q = rng.standard_normal((2, 32)) * 3
    out = _one_seq(k, v, q)
    np.testing.assert_allclose(out, np.tile(v[0].astype(np.float64), (2, 1)), atol=1e-13)


@pytest.mark.parametrize("a", [-3.0, 0.5, 2.0, 11.0])
def test_two_token_sigmoid_pins_scale_and_sign(a):
    """Two tokens with scores a*scale and 0 and values 1 and 0: the output
    is the logistic function of a/sqrt(D)."""
    D = 16
    q = np.zeros((1, D)); q[0, 0] = 1.0
    k = np.zeros((2, 1, D)); k[0, 0, 0] = a
    v = np.zeros((2, 1, D)); v[0, 0, :] = 1.0
    out = _one_seq(k, v, q)
    expect = 1.0 / (1.0 + math.exp(-a / math.sqrt(D)))
    np.testing.assert_allclose(out[0], np.full(D, expect), rtol=0, atol=1e-15)


def test_gqa_query_heads_use_contiguous_kv_groups():
    """Query head hq reads KV head hq // (Hq/Hkv): with values constant per KV
    head the output of hq is that head's constant."""
    rng = np.random.default_rng(4)
    Hq, Hkv, D, ctx = 12, 3, 8, 9
    k = rng.standard_normal((ctx, Hkv, D))
    consts = np.array([1.5, -2.0, 7.0])
    v = np.broadcast_to(consts[None, :, None], (ctx, Hkv, D)).copy()
    q = rng.standard_normal((Hq, D))
    out = _one_seq(k, v, q)
    for hq in range(Hq):
        np.testing.assert_allclose(out[hq], consts[hq // 4], atol=1e-13)


@pytest.mark.parametrize("j", [0, 3, 4, 5, 15, 16, 63])
def test_spike_key_selects_its_value(j):
    """A key equal to c * q/|q| with large c at logical position j takes all
    the weight: the output is V_j (checks per-position addressing)."""
    rng = np.random.default_rng(5 + j)
    ctx, D = 64, 16
    q = rng.standard_normal((1, D))
    k = rng.standard_normal((ctx, 1, D)) * 0.1
    k[j, 0] = 400.0 * q[0] / np.linalg.norm(q[0])
    v = rng.standard_normal((ctx, 1, D)).astype(np.float32)
    out = _one_seq(k, v, q, bs=4, seed=j)
    np.testing.assert_allclose(out[0], v[j, 0].astype(np.float64), atol=1e-12)


# --------------------------------------------------------------------------
# Invariants
# --------------------------------------------------------------------------

def test_block_permutation_invariance():
    """Relabelling physical blocks (moving pages, rewriting tables) leaves
    the output bit-identical: the result depends on logical order only
    (teaching page, "From logical token to physical block")."""
    w = wl.make_workload("tiny_fp32", seed=1)
    out1, f1 = oracle.decode(w.q, w.key_cache, w.value_cache, w.block_tables, w.context_lens)
    perm = np.random.default_rng(9).permutation(w.num_blocks)
    kc = np.empty_like(w.key_cache); vc = np.empty_like(w.value_cache)
    kc[perm] = w.key_cache; vc[perm] = w.value_cache
    bt = np.where(w.block_tables >= 0, perm[np.maximum(w.block_tables, 0)], -1).astype(np.int32)
    out2, f2 = oracle.decode(w.q, kc, vc, bt, w.context_lens)
    assert np.array_equal(out1, out2) and not f1.any() and not f2.any()


def test_nan_poison_outside_context_is_never_read():
    """Unreferenced blocks and slots past each context length hold NaN in
    the workloads; replacing them by zeros must not change a bit
    (optimisation-route page, "What Triton is good for": mask tokens past
    the valid context)."""
    w = wl.make_workload("tiny_fp32", seed=2)
    assert np.isnan(w.key_cache).any()
    out1, f1 = oracle.decode(w.q, w.key_cache, w.value_cache, w.block_tables, w.context_lens)
    out2, f2 = oracle.decode(w.q, np.nan_to_num(w.key_cache, nan=0.0),
                             np.nan_to_num(w.value_cache, nan=0.0), w.block_tables, w.context_lens)
    assert np.all(np.isfinite(out1)) and np.array_equal(out1, out2)


def test_partials_merge_to_single_pass():
    rng_w = wl.custom_workload(dtype=wl.DTYPE_F32, batch=4, num_q_heads=8, num_kv_heads=2,
                               head_dim=16, block_size=4, context_lens=[1, 7, 33, 64], seed=4)
    w = rng_w
    ref, _ = oracle.decode(w.q, w.key_cache, w.value_cache, w.block_tables, w.context_lens)
    for P in (4, 8, 12, 64):
        maxp = -(-64 // P)
        pm, ps, po, f = oracle.partials(w.q, w.key_cache, w.value_cache, w.block_tables,
                                        w.context_lens, P, maxp)
        assert f == 0
        np.testing.assert_allclose(oracle.merge(pm, ps, po), ref, atol=1e-13)
        # empty partitions are (-inf, 0, 0)
        for b, ctx in enumerate(w.context_lens):
            n = -(-int(ctx) // P)
            assert np.all(ps[b, :, n:] == 0) and np.all(np.isneginf(pm[b, :, n:]))
            assert np.all(ps[b, :, :n] >= 1.0)
    # a single partition is the single pass itself
    pm, ps, po, _ = oracle.partials(w.q, w.key_cache, w.value_cache, w.block_tables,
                                    w.context_lens, 64, 1)
    assert np.array_equal(po[:, :, 0], ref)


def test_partial_max_and_sum_closed_form():
    """Two tokens with scores a*scale and 0: max = max(a*scale, 0) and
    sum = 1 + exp(-|a*scale|)."""
    D, a = 16, 6.0
    q = np.zeros((1, 1, D), np.float32); q[0, 0, 0] = 1.0
    kc = np.zeros((2, 2, 1, D), np.float32); kc[1, 0, 0, 0] = a
    vc = np.zeros_like(kc)
    pm, ps, po, f = oracle.partials(q, kc, vc, np.array([[1]], np.int32), np.array([2], np.int32), 2, 1)
    s = a / math.sqrt(D)
    assert pm[0, 0, 0] == pytest.approx(s, abs=1e-15)
    assert ps[0, 0, 0] == pytest.approx(1.0 + math.exp(-s), abs=1e-15)


# --------------------------------------------------------------------------
# Edge cases and flags
# --------------------------------------------------------------------------

def test_zero_context_gives_zeros():
    w = wl.custom_workload(dtype=wl.DTYPE_F32, batch=3, num_q_heads=2, num_kv_heads=1,
                           head_dim=8, block_size=4, context_lens=[0, 5, 0], seed=5)
    out, flags = oracle.decode(w.q, w.key_cache, w.value_cache, w.block_tables, w.context_lens)
    assert not flags.any()
    assert np.all(out[0] == 0) and np.all(out[2] == 0) and np.all(np.isfinite(out[1]))


def test_bad_metadata_is_flagged_and_zeroed():
    w = wl.custom_workload(dtype=wl.DTYPE_F32, batch=3, num_q_heads=2, num_kv_heads=1,
                           head_dim=8, block_size=4, context_lens=[6, 5, 7], seed=6)
    bt = w.block_tables.copy()
    cl = w.context_lens.copy()
    bt[0, 1] = w.num_blocks  # out of range block id
    cl[2] = w.max_blocks * w.block_size + 1  # longer than the table
    out, flags = oracle.decode(w.q, w.key_cache, w.value_cache, bt, cl)
    assert flags[0] == oracle.FLAG_BLOCK_ID and flags[1] == 0 and flags[2] == oracle.FLAG_CONTEXT_LEN
    assert np.all(out[0] == 0) and np.all(out[2] == 0) and np.any(out[1] != 0)
    kc = w.key_cache.copy(); vc = w.value_cache.copy()
    f = oracle.write_kv_cache(kc, vc, np.ones((2, 1, 8), np.float32), np.ones((2, 1, 8), np.float32),
                              np.array([-1, w.num_blocks * w.block_size]))
    assert f == oracle.FLAG_SLOT
    assert np.array_equal(kc, w.key_cache, equal_nan=True)


# ---------------------------------------------------------------------------
# FP8 KV pages (E4M3, OCP 8-bit floating point, "fn" form).  The oracle's
# codec is pinned against torch's float8_e4m3fn (a library decoder), against
# a brute-force nearest-code search, and against values of the format's
# definition; the quantising write against a hand-worked example.
# ---------------------------------------------------------------------------
def test_e4m3_values_of_the_definition():
    v = oracle.e4m3_value(np.array([0x00, 0x01, 0x07, 0x08, 0x38, 0x3F, 0x40, 0x7E, 0x80,
                                    0xB8, 0xFE], dtype=np.uint8))
    assert v.tolist() == [0.0, 2.0 ** -9, 7 * 2.0 ** -9, 2.0 ** -6, 1.0, 1.875, 2.0, 448.0,
                          -0.0, -1.0, -448.0]
    assert np.isnan(oracle.e4m3_value(np.array([0x7F, 0xFF], dtype=np.uint8))).all()
    pos = oracle.e4m3_value(np.arange(0x7F, dtype=np.uint8))
    assert np.all(np.diff(pos) > 0), "codes 0x00..0x7E increase"


def test_e4m3_values_match_torch_float8():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_value(codes)
    theirs = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(theirs))
    ok = ~np.isnan(ours)
    assert np.array_equal(ours[ok], theirs[ok])
    assert np.array_equal(np.signbit(ours[ok]), np.signbit(theirs[ok]))


def _nearest_code_brute(x: float) -> int:
    codes = np.arange(256, dtype=np.uint8)
    vals = oracle.e4m3_value(codes)
    finite = ~np.isnan(vals)
    if abs(x) >= 448.0:
        return 0x7E | (0x80 if np.signbit(x) else 0)
    d = np.where(finite, np.abs(vals - x), np.inf)
    best = np.flatnonzero(d == d.min())
    # equal distance: the code whose mantissa (its last bit) is even; the
    # two zeros are equally near only to 0 itself: keep x's sign
    best = [int(c) for c in best if not (vals[c] == 0 and np.signbit(vals[c]) != np.signbit(x))]
    even = [c for c in best if c % 2 == 0]
    return (even or best)[0]


def test_e4m3_encode_is_the_nearest_code():
    rng = np.random.default_rng(7)
    xs = np.concatenate([rng.normal(0, 4, 300), rng.normal(0, 0.01, 200),
                         rng.uniform(-500, 500, 100), [0.0, -0.0, 447.9, 448.0, 449.0, 479.9]])
    # every midpoint between neighbouring codes (ties)
    pos = oracle.e4m3_value(np.arange(0x7F, dtype=np.uint8))
    mids = (pos[1:] + pos[:-1]) / 2
    xs = np.concatenate([xs, mids, -mids])
    got = oracle.e4m3_encode(xs)
    want = np.array([_nearest_code_brute(float(x)) for x in xs], dtype=np.uint8)
    assert np.array_equal(got, want)
    assert oracle.e4m3_encode(np.array([np.nan]))[0] == 0x7F


def test_decode_fp8_matches_sdpa_on_torch_float8_values():
    """decode over FP8 pages == torch's float64 SDPA on K/V that torch's own
    float8_e4m3fn conversion decodes, times the per-tensor scales, gathered
    here by plain indexing through the table (pins the dequantisation, the
    scales' roles and the bf16 query path of decode_fp8)."""
    lens = [1, 6, 11]
    w = wl.custom_workload(dtype=wl.DTYPE_FP8, batch=3, num_q_heads=8, num_kv_heads=2,
                           head_dim=32, block_size=4, context_lens=lens, seed=9,
                           k_scale=0.25, v_scale=0.5)
    out, fl = oracle.decode_fp8(w.q, w.key_cache, w.value_cache, w.k_scale, w.v_scale,
                                w.block_tables, w.context_lens)
    assert not fl.any()
    as_f8 = lambda a: torch.from_numpy(a).view(torch.float8_e4m3fn).to(torch.float64)
    for b, n in enumerate(lens):
        rows = [(w.block_tables[b, t // 4], t % 4) for t in range(n)]
        K = torch.stack([as_f8(w.key_cache[pb, off]) for pb, off in rows]) * 0.25
        V = torch.stack([as_f8(w.value_cache[pb, off]) for pb, off in rows]) * 0.5
        qb = torch.from_numpy(w.q[b].copy()).view(torch.bfloat16).to(torch.float64)
        ref = torch.nn.functional.scaled_dot_product_attention(
            qb.reshape(1, 8, 1, 32), K.permute(1, 0, 2)[None], V.permute(1, 0, 2)[None],
            scale=1.0 / math.sqrt(32), enable_gqa=True).reshape(8, 32).numpy()
        np.testing.assert_allclose(out[b], ref, rtol=0, atol=1e-12)
    # swapping the scales changes the result: each scale belongs to its tensor
    swapped, _ = oracle.decode_fp8(w.q, w.key_cache, w.value_cache, w.v_scale, w.k_scale,
                                   w.block_tables, w.context_lens)
    assert np.abs(swapped[1:] - out[1:]).max() > 1e-3


def test_write_kv_cache_fp8_worked_example():
    """Two tokens into a 2-block pool of 2-token pages, 1 KV head, head_dim 4:
    bf16 1.0, -3.0, 0.25, 1000.0 divided by k_scale 0.5 are 2, -6, 0.5 and
    2000 -> codes 0x40, 0xCC (-1.5 * 2^2: exponent field 9, mantissa 4),
    0x30, 0x7E (saturated); V by v_scale 2.0."""
    def bf16(xs):
        return (np.array(xs, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)
    kc = np.zeros((2, 2, 1, 4), dtype=np.uint8)
    vc = np.zeros_like(kc)
    k_new = bf16([[1.0, -3.0, 0.25, 1000.0], [0.0, 0.0, 0.0, 0.0]]).reshape(2, 1, 4)
    v_new = bf16([[1.0, 2.0, 3.0, 4.0], [0.5, 0.5, 0.5, 0.5]]).reshape(2, 1, 4)
    f = oracle.write_kv_cache_fp8(kc, vc, k_new, v_new, np.array([3, -1]), 0.5, 2.0)
    assert f == 0
    assert kc[1, 1, 0].tolist() == [0x40, 0xCC, 0x30, 0x7E]
    # 0.5, 1, 1.5, 2 -> 0x30, 0x38, 0x3C, 0x40
    assert vc[1, 1, 0].tolist() == [0x30, 0x38, 0x3C, 0x40]
    assert not kc[0].any() and not kc[1, 0].any()
    assert oracle.write_kv_cache_fp8(kc, vc, k_new, v_new, np.array([4, 0]), 0.5, 2.0) == \
        oracle.FLAG_SLOT


# ---------------------------------------------------------------------------
# Paged (chunked) prefill with the causal mask (next-row groundwork: the
# oracle comes before any kernel).  Pinned against torch's causal SDPA on
# K/V gathered here by plain indexing, and by invariants.
# ---------------------------------------------------------------------------
def _prompt_case(lens, seed, Hq=8, Hkv=2, D=32, bs=4):
    w = wl.custom_workload(dtype=wl.DTYPE_F32, batch=len(lens), num_q_heads=Hq,
                           num_kv_heads=Hkv, head_dim=D, block_size=bs, context_lens=lens,
                           seed=seed)
    rng = np.random.default_rng(seed + 100)
    q = rng.standard_normal((int(sum(lens)), Hq, D)).astype(np.float32)
    qs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return w, q, qs


def _rows_by_table(cache, table, n, bs):
    return np.stack([cache[table[t // bs], t % bs] for t in range(n)]).astype(np.float64)


def test_prefill_matches_torch_causal_sdpa():
    lens = [11, 7, 1]
    w, q, qs = _prompt_case(lens, seed=3)
    out, fl = oracle.prefill(q, w.key_cache, w.value_cache, w.block_tables, w.context_lens, qs)
    assert not fl.any()
    D = w.head_dim
    for b, n in enumerate(lens):
        K = _rows_by_table(w.key_cache, w.block_tables[b], n, w.block_size)
        V = _rows_by_table(w.value_cache, w.block_tables[b], n, w.block_size)
        qt = torch.from_numpy(q[qs[b]:qs[b + 1]].astype(np.float64)).permute(1, 0, 2)[None]
        kt = torch.from_numpy(K).permute(1, 0, 2)[None]
        vt = torch.from_numpy(V).permute(1, 0, 2)[None]
        ref = torch.nn.functional.scaled_dot_product_attention(
            qt, kt, vt, is_causal=True, scale=1.0 / math.sqrt(D), enable_gqa=True)
        ref = ref[0].permute(1, 0, 2).numpy()
        assert np.allclose(out[qs[b]:qs[b + 1]], ref, rtol=0, atol=1e-12)


def test_prefill_in_chunks_equals_one_shot():
    lens = [13, 9]
    w, q, qs = _prompt_case(lens, seed=4)
    full, _ = oracle.prefill(q, w.key_cache, w.value_cache, w.block_tables, w.context_lens, qs)
    cut = [5, 9]  # the second sequence has nothing left for chunk 2
    q1 = np.concatenate([q[qs[b]:qs[b] + cut[b]] for b in range(2)])
    q2 = np.concatenate([q[qs[b] + cut[b]:qs[b + 1]] for b in range(2)])
    qs1 = np.array([0, cut[0], cut[0] + cut[1]], dtype=np.int32)
    rest = [lens[b] - cut[b] for b in range(2)]
    qs2 = np.array([0, rest[0], rest[0] + rest[1]], dtype=np.int32)
    o1, f1 = oracle.prefill(q1, w.key_cache, w.value_cache, w.block_tables,
                            np.array(cut, dtype=np.int32), qs1)
    o2, f2 = oracle.prefill(q2, w.key_cache, w.value_cache, w.block_tables, w.context_lens, qs2)
    assert not f1.any() and not f2.any()
    for b in range(2):
        assert np.array_equal(o1[qs1[b]:qs1[b + 1]], full[qs[b]:qs[b] + cut[b]])
        assert np.array_equal(o2[qs2[b]:qs2[b + 1]], full[qs[b] + cut[b]:qs[b + 1]])


def test_prefill_last_token_is_decode_and_first_is_v0():
    lens = [10, 6]
    w, q, qs = _prompt_case(lens, seed=5)
    out, _ = oracle.prefill(q, w.key_cache, w.value_cache, w.block_tables, w.context_lens, qs)
    last = np.stack([q[qs[b + 1] - 1] for b in range(2)])
    dec, _ = oracle.decode(last, w.key_cache, w.value_cache, w.block_tables, w.context_lens,
                           1.0 / math.sqrt(w.head_dim))
    group = w.num_q_heads // w.num_kv_heads
    for b in range(2):
        assert np.array_equal(out[qs[b + 1] - 1], dec[b])
        # the first prompt token sees only itself: out = V_0 of its KV head
        v0 = w.value_cache[w.block_tables[b, 0], 0].astype(np.float64)
        for hq in range(w.num_q_heads):
            assert np.array_equal(out[qs[b], hq], v0[hq // group])


def test_prefill_is_causal():
    """NaN in every slot after position p leaves the rows up to p unchanged."""
    lens = [12]
    w, q, qs = _prompt_case(lens, seed=6)
    out, _ = oracle.prefill(q, w.key_cache, w.value_cache, w.block_tables, w.context_lens, qs)
    p = 6
    kc, vc = w.key_cache.copy(), w.value_cache.copy()
    for t in range(p + 1, lens[0]):
        pb, off = w.block_tables[0, t // w.block_size], t % w.block_size
        kc[pb, off] = np.nan
        vc[pb, off] = np.nan
    out2, _ = oracle.prefill(q, kc, vc, w.block_tables, w.context_lens, qs)
    assert np.array_equal(out2[:p + 1], out[:p + 1])
    assert np.isnan(out2[p + 1:]).all()


def test_prefill_flags():
    lens = [8, 5]
    w, q, qs = _prompt_case(lens, seed=7)
    cl = np.array([8, 3], dtype=np.int32)  # sequence 1: 5 new tokens but a 3-token history
    out, fl = oracle.prefill(q, w.key_cache, w.value_cache, w.block_tables, cl, qs)
    assert fl.tolist() == [0, oracle.FLAG_CONTEXT_LEN]
    assert not out[qs[1]:].any() and out[:qs[1]].any()
    bt = w.block_tables.copy()
    bt[0, 1] = w.num_blocks + 3
    out, fl = oracle.prefill(q, w.key_cache, w.value_cache, bt, w.context_lens, qs)
    assert fl[0] == oracle.FLAG_BLOCK_ID and not out[:qs[1]].any()
