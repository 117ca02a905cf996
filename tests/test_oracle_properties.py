"""Property-based pins of the oracle (hypothesis): over random small shapes,
lengths, page sizes and physical placements, the oracle must satisfy what
the pages and the mathematics fix -- paged attention equals attention on the
same K/V stored contiguously (teaching page, "From logical token to physical
block"; computed here by torch's float64 SDPA on rows gathered by plain
indexing), split partials merged with the running-max rule equal the single
pass (route page, "The core idea of high-performance PagedAttention"), a
chunked prefill equals the one-shot prefill, and a slot write is read back
where the block table says.  Host only."""
import math

import numpy as np
import torch
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle

SETTINGS = settings(max_examples=30, deadline=None, derandomize=True)


@st.composite
def paged_case(draw):
    """A random pool: heads, head_dim, page size, lengths (0 allowed), and
    tables that scatter every sequence's pages over a shuffled pool with NaN
    in every slot no context reaches."""
    hkv = draw(st.sampled_from([1, 2, 4]))
    group = draw(st.sampled_from([1, 2, 3, 8]))
    D = draw(st.sampled_from([4, 8, 16]))
    bs = draw(st.sampled_from([1, 2, 4, 8]))
    lens = draw(st.lists(st.integers(0, 40), min_size=1, max_size=4))
    seed = draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    B = len(lens)
    pages = [-(-n // bs) for n in lens]
    MB = max(pages + [1])
    NB = sum(pages) + draw(st.integers(0, 5)) + 1
    perm = rng.permutation(NB).astype(np.int32)
    tables = np.full((B, MB), -1, dtype=np.int32)
    contig_k, contig_v = [], []
    kc = np.full((NB, bs, hkv, D), np.nan, dtype=np.float32)
    vc = np.full_like(kc, np.nan)
    at = 0
    for b, n in enumerate(lens):
        tables[b, :pages[b]] = perm[at:at + pages[b]]
        at += pages[b]
        k = rng.standard_normal((n, hkv, D)).astype(np.float32)
        v = rng.standard_normal((n, hkv, D)).astype(np.float32)
        for t in range(n):
            kc[tables[b, t // bs], t % bs] = k[t]
            vc[tables[b, t // bs], t % bs] = v[t]
        contig_k.append(k)
        contig_v.append(v)
    q = rng.standard_normal((B, hkv * group, D)).astype(np.float32)
    return dict(q=q, kc=kc, vc=vc, tables=tables, lens=np.array(lens, dtype=np.int32),
                k=contig_k, v=contig_v, hkv=hkv, group=group, D=D, bs=bs)


def _sdpa(q, k, v, scale):
    """torch float64 SDPA of one query row set over contiguous K/V (GQA)."""
    n, hkv, D = k.shape
    hq = q.shape[0]
    if n == 0:
        return np.zeros((hq, D))
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q.astype(np.float64)).reshape(1, hq, 1, D),
        torch.from_numpy(k.astype(np.float64)).permute(1, 0, 2)[None],
        torch.from_numpy(v.astype(np.float64)).permute(1, 0, 2)[None],
        scale=scale, enable_gqa=True).reshape(hq, D).numpy()


@SETTINGS
@given(paged_case())
def test_paged_decode_equals_contiguous_attention(c):
    scale = 1.0 / math.sqrt(c["D"])
    out, flags = oracle.decode(c["q"], c["kc"], c["vc"], c["tables"], c["lens"], scale)
    assert not flags.any()
    for b in range(len(c["lens"])):
        ref = _sdpa(c["q"][b], c["k"][b], c["v"][b], scale)
        np.testing.assert_allclose(out[b], ref, rtol=0, atol=1e-12)


@SETTINGS
@given(paged_case(), st.sampled_from([1, 2, 3, 5, 8, 64]))
def test_partials_merge_to_the_single_pass(c, part):
    scale = 1.0 / math.sqrt(c["D"])
    P = max(1, -(-int(c["lens"].max()) // part))
    pm, ps, po, flags = oracle.partials(c["q"], c["kc"], c["vc"], c["tables"], c["lens"], part,
                                        P, scale)
    assert flags == 0
    merged = oracle.merge(pm, ps, po)
    single, _ = oracle.decode(c["q"], c["kc"], c["vc"], c["tables"], c["lens"], scale)
    np.testing.assert_allclose(merged, single, rtol=0, atol=1e-12)
    # empty partitions carry (-inf, 0, 0)
    for b, n in enumerate(c["lens"]):
        for p in range(-(-int(n) // part), P):
            assert np.all(pm[b, :, p] == -np.inf) and not ps[b, :, p].any()


@SETTINGS
@given(paged_case(), st.data())
def test_chunked_prefill_equals_one_shot(c, data):
    """Whole prompts at once, or in two chunks at a random cut per sequence:
    the same rows."""
    lens = c["lens"]
    scale = 1.0 / math.sqrt(c["D"])
    rng = np.random.default_rng(int(lens.sum()) + 7)
    T = int(lens.sum())
    hq = c["hkv"] * c["group"]
    q = rng.standard_normal((T, hq, c["D"])).astype(np.float32)
    qs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    full, flags = oracle.prefill(q, c["kc"], c["vc"], c["tables"], lens, qs, scale)
    assert not flags.any()
    cut = [data.draw(st.integers(0, int(n))) for n in lens]
    first = np.concatenate([q[qs[b]:qs[b] + cut[b]] for b in range(len(lens))])
    second = np.concatenate([q[qs[b] + cut[b]:qs[b + 1]] for b in range(len(lens))])
    qs1 = np.concatenate([[0], np.cumsum(cut)]).astype(np.int32)
    rest = [int(n) - k for n, k in zip(lens, cut)]
    qs2 = np.concatenate([[0], np.cumsum(rest)]).astype(np.int32)
    o1, f1 = oracle.prefill(first, c["kc"], c["vc"], c["tables"], np.array(cut, np.int32), qs1,
                            scale)
    o2, f2 = oracle.prefill(second, c["kc"], c["vc"], c["tables"], lens, qs2, scale)
    assert not f1.any() and not f2.any()
    for b in range(len(lens)):
        assert np.array_equal(o1[qs1[b]:qs1[b + 1]], full[qs[b]:qs[b] + cut[b]])
        assert np.array_equal(o2[qs2[b]:qs2[b + 1]], full[qs[b] + cut[b]:qs[b + 1]])
    # each sequence's last prompt row is its decode
    last = np.stack([q[qs[b + 1] - 1] if lens[b] else np.zeros((hq, c["D"]), np.float32)
                     for b in range(len(lens))])
    dec, _ = oracle.decode(last, c["kc"], c["vc"], c["tables"], lens, scale)
    for b in range(len(lens)):
        if lens[b]:
            assert np.array_equal(full[qs[b + 1] - 1], dec[b])


@SETTINGS
@given(paged_case(), st.integers(0, 2**31 - 1))
def test_slot_write_is_read_back_through_the_table(c, seed):
    """Write a fresh row into the slot of one random (sequence, position):
    the gather through the table returns it there and nothing else moves."""
    lens = c["lens"]
    live = [b for b in range(len(lens)) if lens[b] > 0]
    if not live:
        return
    rng = np.random.default_rng(seed)
    b = live[rng.integers(len(live))]
    t = int(rng.integers(lens[b]))
    bs = c["bs"]
    slot = np.array([c["tables"][b, t // bs] * bs + t % bs], dtype=np.int64)
    kn = rng.standard_normal((1, c["hkv"], c["D"])).astype(np.float32)
    vn = rng.standard_normal((1, c["hkv"], c["D"])).astype(np.float32)
    kc, vc = c["kc"].copy(), c["vc"].copy()
    assert oracle.write_kv_cache(kc, vc, kn, vn, slot) == 0
    keys, values, flags = oracle.gather_kv(kc, vc, c["tables"][b], int(lens[b]))
    assert flags == 0
    expect_k = c["k"][b].astype(np.float64)
    expect_v = c["v"][b].astype(np.float64)
    expect_k[t] = kn[0]
    expect_v[t] = vn[0]
    assert np.array_equal(keys, expect_k) and np.array_equal(values, expect_v)
