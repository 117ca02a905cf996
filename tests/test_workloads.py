"""The seeded input generators: determinism and the structure each workload
recipe promises (host only, no attention arithmetic involved)."""
import numpy as np
import pytest

from paged_kv_cache_334_b200 import workloads as wl


def test_tiny_recipe():
    w = wl.make_workload("tiny_fp32", seed=0)
    assert (w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, w.num_blocks) == (3, 4, 4, 64, 4, 16)
    assert list(w.context_lens) == [5, 9, 12]
    assert list(w.block_tables[0]) == [7, 2, 9]
    rest = np.concatenate([w.block_tables[1], w.block_tables[2]])
    assert len(set(rest.tolist())) == 6 and not set(rest.tolist()) & {7, 2, 9}
    assert w.q.dtype == np.float32 and w.key_cache.shape == (16, 4, 4, 64)
    assert w.slot_mapping is None


def test_determinism_and_seed_dependence():
    a = wl.make_workload("gqa_bf16", seed=3, batch=4)
    b = wl.make_workload("gqa_bf16", seed=3, batch=4)
    c = wl.make_workload("gqa_bf16", seed=4, batch=4)
    for f in ("q", "key_cache", "value_cache", "block_tables", "context_lens", "k_new", "slot_mapping"):
        assert np.array_equal(getattr(a, f), getattr(b, f))
    assert not np.array_equal(a.context_lens, c.context_lens)


@pytest.mark.parametrize("name,batch", [("gqa_bf16", 8), ("mixed_bf16", 6), ("long_bf16", 1),
                                        ("mqa_prefix_bf16", 8)])
def test_structure(name, batch):
    w = wl.make_workload(name, seed=0, batch=batch)
    bs = w.block_size
    assert w.dtype == wl.DTYPE_BF16 and w.q.dtype == np.uint16
    pages = [(-(-int(c) // bs)) for c in w.context_lens]
    assert max(pages) <= w.max_blocks
    used = []
    for b in range(w.batch):
        row = w.block_tables[b]
        assert np.all(row[:pages[b]] >= 0) and np.all(row[:pages[b]] < w.num_blocks)
        assert np.all(row[pages[b]:] == -1)
        used.extend(row[:pages[b]].tolist())
    if name == "mqa_prefix_bf16":
        prefix = w.block_tables[:, :64]
        assert np.all(prefix == prefix[0])
        assert np.all(w.context_lens >= 2049) and np.all(w.context_lens <= 3072)
        suffix_blocks = [x for b in range(w.batch) for x in w.block_tables[b, 64:pages[b]]]
        assert len(set(suffix_blocks)) == len(suffix_blocks)
    else:
        assert len(set(used)) == len(used)  # private pages
    if name == "gqa_bf16":
        assert np.all(w.context_lens >= 128) and np.all(w.context_lens <= 2048)
    if name == "mixed_bf16":
        assert all(any(0 <= c - x <= 15 for x in (128, 4096, 16000)) for c in w.context_lens)
    if name == "long_bf16":
        assert np.all(w.context_lens == 131072) and w.partition_tokens == 512
    # the newest token's slot is reserved and poisoned until written
    assert w.slot_mapping is not None and len(w.slot_mapping) == w.batch
    nan_bits = 0x7FC0
    for i, b in enumerate(range(w.batch)):
        t = int(w.context_lens[b]) - 1
        pb, off = int(w.block_tables[b, t // bs]), t % bs
        assert w.slot_mapping[i] == pb * bs + off
        assert np.all(w.key_cache[pb, off] == nan_bits)
        assert not np.any(w.k_new[i] == nan_bits)


def test_poison_marks_exactly_the_invisible_slots():
    w = wl.make_workload("tiny_fp32", seed=0)
    live = np.zeros((w.num_blocks, w.block_size), bool)
    for b in range(w.batch):
        for t in range(int(w.context_lens[b])):
            live[w.block_tables[b, t // w.block_size], t % w.block_size] = True
    nan_slot = np.isnan(w.key_cache).all(axis=(2, 3))
    assert np.array_equal(nan_slot, ~live)
    assert np.array_equal(np.isnan(w.value_cache).all(axis=(2, 3)), ~live)


def test_roofline_bytes_counts_shared_prefix_once():
    w = wl.make_workload("mqa_prefix_bf16", seed=0, batch=4)
    row = w.num_kv_heads * w.head_dim * 2
    kv_unique = 2 * row * (2048 + int(sum(w.context_lens - 2048)))
    qo = 2 * w.batch * w.num_q_heads * w.head_dim * 2
    meta = w.block_tables.size * 4 + w.batch * 4
    write = 2 * (w.k_new.nbytes + w.v_new.nbytes) + w.slot_mapping.nbytes
    assert wl.roofline_bytes(w) == kv_unique + qo + meta + write
    assert wl.roofline_bytes(w, include_write=False) == kv_unique + qo + meta


def test_block_size_override_keeps_lengths_and_pages_them_anew():
    """A page-size sweep: the same context lengths, paged with another block
    size, still a consistent allocator (every visible token in its own slot)."""
    base = wl.make_workload("gqa_bf16", seed=2)
    assert base.block_size == 16
    assert wl.make_workload("gqa_bf16", seed=2, block_size=16).block_tables.tolist() == \
        base.block_tables.tolist()
    for bs in (8, 64, 256):
        w = wl.make_workload("gqa_bf16", seed=2, block_size=bs)
        assert w.block_size == bs
        assert w.context_lens.tolist() == base.context_lens.tolist()
        seen = set()
        for b, ctx in enumerate(w.context_lens):
            for t in range(0, int(ctx), 97):
                pb = int(w.block_tables[b, t // bs])
                assert 0 <= pb < w.num_blocks
                key = (pb, t % bs)
                assert key not in seen
                seen.add(key)
    with pytest.raises(ValueError):
        wl.make_workload("gqa_bf16", block_size=48)
    with pytest.raises(ValueError):
        wl.make_workload("mqa_prefix_bf16", block_size=16)


def test_gqa_fp8_pages():
    """gqa_fp8: gqa_bf16's lengths; E4M3 codes with exponent fields 3..9 in
    visible slots, the NaN code everywhere else (the newest tokens' slots
    too, until the write), bf16 q and new rows, and half the cache bytes."""
    w = wl.make_workload("gqa_fp8", seed=1)
    g = wl.make_workload("gqa_bf16", seed=1)
    assert w.context_lens.tolist() == g.context_lens.tolist()
    assert w.key_cache.dtype == np.uint8 and w.q.dtype == np.uint16
    assert w.k_new.dtype == np.uint16 and w.k_new.shape == (w.batch, 8, 128)
    assert (w.k_scale, w.v_scale) == (wl.FP8_K_SCALE, wl.FP8_V_SCALE)
    bs = w.block_size
    live = np.zeros((w.num_blocks, bs), dtype=bool)
    for b, ctx in enumerate(w.context_lens):
        for t in range(int(ctx) - 1):  # the newest token's slot is poisoned too
            live[w.block_tables[b, t // bs], t % bs] = True
    for cache in (w.key_cache, w.value_cache):
        vis = cache[live]
        assert not np.any(vis == 0x7F)
        expo = (vis >> 3) & 15
        assert expo.min() >= 3 and expo.max() <= 9
        assert np.all(cache[~live] == 0x7F)
    for b, ctx in enumerate(w.context_lens):
        t = int(ctx) - 1
        pb, off = w.block_tables[b, t // bs], t % bs
        assert w.slot_mapping[b] == pb * bs + off
    # the cache rows are half as wide as bf16 ones; q, out and new rows are not
    kv_bf16 = wl.roofline_bytes(g, include_write=False)
    kv_fp8 = wl.roofline_bytes(w, include_write=False)
    qo = 2 * w.batch * w.num_q_heads * w.head_dim * 2
    meta = w.block_tables.size * 4 + w.context_lens.size * 4
    assert kv_fp8 - qo - meta == (kv_bf16 - qo - meta) // 2


def test_prefill_inputs_store_every_context_token():
    """Whole prompts over gqa_bf16's pool: the held-back newest tokens are
    back in their slots, every other slot past a context is still NaN."""
    w = wl.make_workload("gqa_bf16", seed=1, batch=6)
    pw = wl.prefill_workload(w, seed=1)
    base = pw.base
    assert base.slot_mapping is None and base.k_new is None
    assert pw.chunk_lens.tolist() == w.context_lens.tolist()
    assert pw.query_start[0] == 0 and np.all(np.diff(pw.query_start) == pw.chunk_lens)
    assert pw.q.shape == (pw.num_tokens, w.num_q_heads, w.head_dim) and pw.q.dtype == np.uint16
    live = np.zeros((base.num_blocks, base.block_size), dtype=bool)
    for b in range(base.batch):
        for t in range(int(base.context_lens[b])):
            live[base.block_tables[b, t // base.block_size], t % base.block_size] = True
    nan = np.uint16(0x7FC0)
    assert not np.any(base.key_cache[live] == nan) and not np.any(base.value_cache[live] == nan)
    assert np.all(base.key_cache[~live] == nan) and np.all(base.value_cache[~live] == nan)
    # the slots the decode step held back now hold exactly its new rows
    for i, s in enumerate(w.slot_mapping.tolist()):
        pb, off = divmod(s, w.block_size)
        assert np.array_equal(base.key_cache[pb, off], w.k_new[i])
        assert np.array_equal(base.value_cache[pb, off], w.v_new[i])
    # the decode workload itself is untouched
    assert np.all(w.key_cache[w.slot_mapping // w.block_size, w.slot_mapping % w.block_size] == nan)


def test_prefill_flops_and_bytes_by_brute_force():
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=4, num_q_heads=8, num_kv_heads=2,
                           head_dim=64, block_size=4, context_lens=[1, 7, 12, 0], seed=3,
                           new_tokens=True)
    for chunk in (None, 5):
        pw = wl.prefill_workload(w, chunk=chunk, seed=2)
        pairs = 0
        for b in range(w.batch):
            ctx, n = int(w.context_lens[b]), int(pw.chunk_lens[b])
            assert n == (ctx if chunk is None else min(ctx, chunk))
            for j in range(n):
                pairs += sum(1 for t in range(ctx) if t <= ctx - n + j)
        assert wl.prefill_flops(pw) == 4 * 64 * 8 * pairs
        kv = 2 * int(w.context_lens.sum()) * 2 * 64 * 2  # no page shared
        qo = 2 * pw.num_tokens * 8 * 64 * 2
        meta = w.block_tables.size * 4 + w.context_lens.size * 4 + pw.query_start.nbytes
        assert wl.prefill_roofline_bytes(pw) == kv + qo + meta
    assert wl.prefill_workload(w, chunk=5).max_query_len == 5
