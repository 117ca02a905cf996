"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Tolerances: address mapping and cache write bit-exact; attention output
<= 1e-5 max-abs for fp32 inputs, <= 2e-2 max-abs and <= 1e-2 mean-abs for
bf16 inputs, against the fp64 oracle on the same seeded inputs.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_334_b200 import pa
from paged_kv_cache_334_b200 import workloads as wl

from _pa_helpers import (assert_close, gpu_write_and_decode, oracle_after_write, to_dev,
                         to_f64, upload)

pytestmark = pytest.mark.gpu


# ---------------------------------------------------------------------------
# Cache write (bit-exact)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", [wl.DTYPE_F32, wl.DTYPE_BF16])
def test_write_kv_cache_bit_exact(dtype):
    rng = np.random.default_rng(11)
    NB, bs, Hkv, D, N = 40, 16, 4, 128, 37
    kc = wl.to_storage(rng.standard_normal((NB, bs, Hkv, D)).astype(np.float32), dtype)
    vc = wl.to_storage(rng.standard_normal((NB, bs, Hkv, D)).astype(np.float32), dtype)
    kn = wl.to_storage(rng.standard_normal((N, Hkv, D)).astype(np.float32), dtype)
    vn = wl.to_storage(rng.standard_normal((N, Hkv, D)).astype(np.float32), dtype)
    slots = rng.choice(NB * bs, size=N, replace=False).astype(np.int64)
    slots[3] = -1  # padding token: skipped
    ok, ov = kc.copy(), vc.copy()
    assert oracle.write_kv_cache(ok, ov, kn, vn, slots) == 0
    dk, dv = to_dev(kc, dtype), to_dev(vc, dtype)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_write_kv_cache(dk, dv, to_dev(kn, dtype), to_dev(vn, dtype),
                         torch.from_numpy(slots).cuda(), err_word=err)
    torch.cuda.synchronize()
    view = torch.uint16 if dtype == wl.DTYPE_BF16 else torch.float32
    gk = dk.view(view).cpu().numpy() if dtype == wl.DTYPE_BF16 else dk.cpu().numpy()
    gv = dv.view(view).cpu().numpy() if dtype == wl.DTYPE_BF16 else dv.cpu().numpy()
    assert gk.tobytes() == ok.tobytes() and gv.tobytes() == ov.tobytes()
    assert int(err.item()) == 0


def test_write_worked_example_slot_9_is_key_cache_2_1():
    """Block size 4, table [7, 2, 9]: token 5's slot is 2*4+1 = 9, i.e.
    key_cache[2, 1] (teaching page, "First define a simple KV cache layout")."""
    NB, bs, Hkv, D = 16, 4, 4, 64
    kc = torch.zeros(NB, bs, Hkv, D, device="cuda")
    vc = torch.zeros_like(kc)
    kn = torch.arange(Hkv * D, dtype=torch.float32, device="cuda").reshape(1, Hkv, D) + 1
    pa.pa_write_kv_cache(kc, vc, kn, -kn, torch.tensor([9], dtype=torch.int64, device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(kc[2, 1], kn[0]) and torch.equal(vc[2, 1], -kn[0])
    kc[2, 1] = 0
    vc[2, 1] = 0
    assert not kc.any() and not vc.any()


def test_write_bad_slot_sets_error_and_skips():
    NB, bs, Hkv, D = 4, 4, 1, 64
    kc = torch.zeros(NB, bs, Hkv, D, device="cuda")
    vc = torch.zeros_like(kc)
    kn = torch.ones(2, Hkv, D, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_write_kv_cache(kc, vc, kn, kn, torch.tensor([NB * bs, -5], device="cuda"),
                         err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == pa.PA_DEVERR_SLOT and not kc.any() and not vc.any()


# ---------------------------------------------------------------------------
# Decode on the five workloads (full size)
# ---------------------------------------------------------------------------

def test_decode_tiny_fp32():
    w = wl.make_workload("tiny_fp32", seed=0)
    d = upload(w)
    out = gpu_write_and_decode(w, d)
    torch.cuda.synchronize()
    ref, flags, _, _ = oracle_after_write(w)
    assert not flags.any()
    assert_close(to_f64(out), ref, w.dtype, "tiny_fp32")


@pytest.mark.parametrize("name", ["gqa_bf16", "mixed_bf16", "mqa_prefix_bf16"])
def test_decode_workload_full_size(name):
    w = wl.make_workload(name, seed=0)
    d = upload(w)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gpu_write_and_decode(w, d, err)
    torch.cuda.synchronize()
    ref, flags, okc, _ = oracle_after_write(w)
    assert not flags.any() and int(err.item()) == 0
    assert_close(to_f64(out), ref, w.dtype, name)
    # the written rows are bit-exact in the device cache
    bs = w.block_size
    pb = torch.from_numpy(w.slot_mapping // bs).cuda()
    off = torch.from_numpy(w.slot_mapping % bs).cuda()
    got = d["key_cache"][pb, off].view(torch.uint16).cpu().numpy()
    assert got.tobytes() == w.k_new.tobytes()


def test_splitk_and_reduce_long_context():
    w = wl.make_workload("long_bf16", seed=0)
    d = upload(w)
    P = w.partition_tokens
    maxp = -(-w.max_blocks * w.block_size // P)
    B, Hq, D = w.batch, w.num_q_heads, w.head_dim
    pm = torch.full((B, Hq, maxp), float("nan"), device="cuda")
    ps = torch.full_like(pm, float("nan"))
    po = torch.full((B, Hq, maxp, D), float("nan"), device="cuda")
    pa.pa_write_kv_cache(d["key_cache"], d["value_cache"], d["k_new"], d["v_new"],
                         d["slot_mapping"])
    pa.pa_decode_splitk(d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                        d["context_lens"], P, pm, ps, po)
    out = torch.empty_like(d["q"])
    pa.pa_reduce(out, pm, ps, po, d["context_lens"], P)
    torch.cuda.synchronize()
    kc, vc = w.key_cache.copy(), w.value_cache.copy()
    oracle.write_kv_cache(kc, vc, w.k_new, w.v_new, w.slot_mapping)
    rm, rs, ro, f = oracle.partials(w.q, kc, vc, w.block_tables, w.context_lens, P, maxp)
    assert f == 0
    np.testing.assert_allclose(to_f64(pm), rm, rtol=0, atol=1e-4)
    np.testing.assert_allclose(to_f64(ps), rs, rtol=1e-4, atol=0)
    np.testing.assert_allclose(to_f64(po), ro, rtol=0, atol=1e-3)
    ref = oracle.merge(rm, rs, ro)
    assert_close(to_f64(out), ref, w.dtype, "long_bf16")
    # pa_decode on the same long inputs agrees too
    out2 = torch.empty_like(d["q"])
    pa.pa_decode(out2, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                 d["context_lens"])
    torch.cuda.synchronize()
    assert_close(to_f64(out2), ref, w.dtype, "long_bf16 pa_decode")


# ---------------------------------------------------------------------------
# Edge cases: boundary lengths, head groups, dtypes, head dims, block sizes
# ---------------------------------------------------------------------------

EDGE_CASES = [
    # dtype, Hq, Hkv, D, bs
    (wl.DTYPE_F32, 4, 4, 64, 4),
    (wl.DTYPE_F32, 8, 2, 128, 16),
    (wl.DTYPE_BF16, 32, 8, 128, 16),
    (wl.DTYPE_BF16, 16, 2, 64, 8),
    (wl.DTYPE_BF16, 64, 1, 128, 32),
    (wl.DTYPE_F32, 16, 16, 128, 1),
    (wl.DTYPE_BF16, 12, 4, 128, 64),
    (wl.DTYPE_BF16, 6, 1, 64, 256),
]


@pytest.mark.parametrize("dtype,Hq,Hkv,D,bs", EDGE_CASES)
def test_boundary_context_lengths(dtype, Hq, Hkv, D, bs):
    """Lengths 0, 1, bs-1, bs, bs+1, several blocks and around the 256-token
    partition edges in one ragged batch (optimisation-route page, "Guard
    correctness before writing the fast version")."""
    lens = sorted({0, 1, max(bs - 1, 1), bs, bs + 1, 3 * bs, 255, 256, 257, 511, 512, 513, 1000})
    w = wl.custom_workload(dtype=dtype, batch=len(lens), num_q_heads=Hq, num_kv_heads=Hkv,
                           head_dim=D, block_size=bs, context_lens=lens, seed=bs + Hq,
                           new_tokens=True)
    d = upload(w)
    out = gpu_write_and_decode(w, d)
    torch.cuda.synchronize()
    ref, flags, _, _ = oracle_after_write(w)
    assert not flags.any()
    got = to_f64(out)
    assert_close(got, ref, dtype, f"{dtype} Hq{Hq} Hkv{Hkv} D{D} bs{bs}")
    assert np.all(got[np.asarray(lens) == 0] == 0)


@pytest.mark.parametrize("group", [1, 2, 3, 4, 5, 8, 12, 16, 64, 128])
def test_group_sizes(group):
    Hkv = 2 if group < 64 else 1
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=5, num_q_heads=group * Hkv,
                           num_kv_heads=Hkv, head_dim=128, block_size=16,
                           context_lens=[1, 17, 300, 777, 2049], seed=group, new_tokens=True)
    d = upload(w)
    out = gpu_write_and_decode(w, d)
    torch.cuda.synchronize()
    ref, _, _, _ = oracle_after_write(w)
    assert_close(to_f64(out), ref, w.dtype, f"group {group}")


def test_splitk_single_partition_matches_decode():
    w = wl.custom_workload(dtype=wl.DTYPE_F32, batch=4, num_q_heads=8, num_kv_heads=2,
                           head_dim=64, block_size=16, context_lens=[5, 64, 200, 256], seed=3)
    d = upload(w)
    B, Hq, D = w.batch, w.num_q_heads, w.head_dim
    pm = torch.empty(B, Hq, 1, device="cuda")
    ps = torch.empty_like(pm)
    po = torch.empty(B, Hq, 1, D, device="cuda")
    pa.pa_decode_splitk(d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                        d["context_lens"], 256, pm, ps, po)
    out = torch.empty_like(d["q"])
    pa.pa_decode(out, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                 d["context_lens"])
    torch.cuda.synchronize()
    np.testing.assert_allclose(po[:, :, 0].cpu().numpy(), out.cpu().numpy(), rtol=0, atol=1e-6)
    ref, _, _, _ = oracle_after_write(w)
    assert_close(to_f64(out), ref, w.dtype, "single partition")


# ---------------------------------------------------------------------------
# Invariants, determinism, workspace
# ---------------------------------------------------------------------------

def test_block_permutation_gives_bit_identical_output():
    w = wl.make_workload("gqa_bf16", seed=5, batch=8)
    d = upload(w)
    out1 = gpu_write_and_decode(w, d)
    perm = np.random.default_rng(1).permutation(w.num_blocks)
    kc = np.empty_like(w.key_cache); vc = np.empty_like(w.value_cache)
    kc[perm] = w.key_cache; vc[perm] = w.value_cache
    w2 = wl.Workload(**{**w.__dict__})
    w2.key_cache, w2.value_cache = kc, vc
    w2.block_tables = np.where(w.block_tables >= 0, perm[np.maximum(w.block_tables, 0)],
                               -1).astype(np.int32)
    sm = w.slot_mapping
    w2.slot_mapping = (perm[sm // w.block_size] * w.block_size + sm % w.block_size).astype(np.int64)
    d2 = upload(w2)
    out2 = gpu_write_and_decode(w2, d2)
    torch.cuda.synchronize()
    assert torch.equal(out1.view(torch.uint16), out2.view(torch.uint16))


def test_repeatable_with_a_reused_workspace():
    """One workspace, zero-filled once, serves repeated calls: identical bits
    every time, whatever the previous call left in it."""
    w = wl.make_workload("mixed_bf16", seed=2, batch=16)
    d = upload(w)
    ws = pa.decode_workspace(d["key_cache"], w.batch, w.num_q_heads, w.max_blocks)
    ws.zero_()
    out1 = gpu_write_and_decode(w, d)
    outs = []
    for _ in range(3):
        o = torch.empty_like(out1)
        pa.pa_decode(o, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                     d["context_lens"], workspace=ws)
        outs.append(o)
    torch.cuda.synchronize()
    for o in outs:
        assert torch.equal(out1.view(torch.uint16), o.view(torch.uint16))


def test_non_default_stream():
    w = wl.make_workload("gqa_bf16", seed=7, batch=4)
    d = upload(w)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out = torch.empty_like(d["q"])
        pa.pa_write_kv_cache(d["key_cache"], d["value_cache"], d["k_new"], d["v_new"],
                             d["slot_mapping"], stream=s)
        pa.pa_decode(out, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                     d["context_lens"], stream=s)
    s.synchronize()
    ref, _, _, _ = oracle_after_write(w)
    assert_close(to_f64(out), ref, w.dtype, "stream")


@pytest.mark.parametrize("j", [0, 255, 256, 511, 512, 65535, 131071])
def test_spike_key_selects_value_at_long_context(j):
    """A key aligned with q at logical position j of a 131072-token history
    takes all the weight: the output is V_j (per-position addressing where a
    tolerance alone could not see one dropped token)."""
    L, D, bs = 131072, 128, 16
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=1, num_q_heads=4, num_kv_heads=1,
                           head_dim=D, block_size=bs, context_lens=[L], seed=j, slack=0.0)
    q = np.zeros((1, 4, D), np.float32)
    q[0, :, 0] = 1.0
    w.q = wl.to_storage(q, wl.DTYPE_BF16)
    pb, off = int(w.block_tables[0, j // bs]), j % bs
    kspike = np.zeros((D,), np.float32)
    kspike[0] = 256.0
    w.key_cache[pb, off, 0] = wl.to_storage(kspike, wl.DTYPE_BF16)
    d = upload(w)
    out = torch.empty_like(d["q"])
    pa.pa_decode(out, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                 d["context_lens"])
    torch.cuda.synchronize()
    vj = oracle.widen(w.value_cache[pb, off, 0])
    got = to_f64(out)[0]
    for hq in range(4):
        np.testing.assert_allclose(got[hq], vj, rtol=0, atol=2e-2)


# ---------------------------------------------------------------------------
# Device-side error reporting (no trap, status word + zero output)
# ---------------------------------------------------------------------------

def test_bad_metadata_sets_error_word_and_zeroes_sequence():
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=4, num_q_heads=8, num_kv_heads=2,
                           head_dim=128, block_size=16, context_lens=[40, 600, 300, 33],
                           seed=9, max_blocks=40)
    bt = w.block_tables.copy()
    cl = w.context_lens.copy()
    bt[0, 1] = w.num_blocks + 5       # visible page with an out-of-range block id
    bt[1, 30] = -7                    # visible page (token 480..495) with a negative id
    bt[3, 10] = 123456789             # entry past ceil(ctx/bs): never read
    cl[2] = 40 * 16 + 1               # longer than the table allows
    d = upload(w)
    d["block_tables"] = torch.from_numpy(bt).cuda()
    d["context_lens"] = torch.from_numpy(cl).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(d["q"])
    pa.pa_decode(out, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                 d["context_lens"], err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == pa.PA_DEVERR_BLOCK_ID | pa.PA_DEVERR_CONTEXT_LEN
    got = to_f64(out)
    assert np.all(got[0] == 0) and np.all(got[1] == 0) and np.all(got[2] == 0)
    ref, flags = oracle.decode(w.q, w.key_cache, w.value_cache, bt, cl)
    assert list(flags) == [oracle.FLAG_BLOCK_ID, oracle.FLAG_BLOCK_ID, oracle.FLAG_CONTEXT_LEN, 0]
    assert_close(got, ref, w.dtype, "bad metadata")
    # split-K path reports the same
    err.zero_()
    maxp = -(-40 * 16 // 256)
    pm = torch.empty(4, 8, maxp, device="cuda"); ps = torch.empty_like(pm)
    po = torch.empty(4, 8, maxp, 128, device="cuda")
    pa.pa_decode_splitk(d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                        d["context_lens"], 256, pm, ps, po, err_word=err)
    out2 = torch.empty_like(out)
    pa.pa_reduce(out2, pm, ps, po, d["context_lens"], 256, err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == pa.PA_DEVERR_BLOCK_ID | pa.PA_DEVERR_CONTEXT_LEN
    assert_close(to_f64(out2), ref, w.dtype, "bad metadata split-K")


def test_negative_context_len_is_flagged():
    w = wl.custom_workload(dtype=wl.DTYPE_F32, batch=2, num_q_heads=4, num_kv_heads=4,
                           head_dim=64, block_size=4, context_lens=[7, 9], seed=1)
    d = upload(w)
    d["context_lens"] = torch.tensor([-3, 9], dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full_like(d["q"], float("nan"))
    pa.pa_decode(out, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                 d["context_lens"], err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == pa.PA_DEVERR_CONTEXT_LEN
    assert torch.all(out[0] == 0) and torch.all(torch.isfinite(out[1]))


# ---------------------------------------------------------------------------
# The persistent page-stream kernel (KV heads 4 or 8, group 1/2/4/8): shapes,
# many sequences with empties, fewer pages than CTAs, long splits.
# ---------------------------------------------------------------------------

STREAM_SHAPES = [
    # dtype, Hq, Hkv, D, bs
    (wl.DTYPE_BF16, 8, 8, 128, 16),
    (wl.DTYPE_BF16, 16, 8, 128, 16),
    (wl.DTYPE_BF16, 64, 8, 128, 16),
    (wl.DTYPE_F32, 32, 8, 128, 16),
    (wl.DTYPE_BF16, 32, 8, 64, 32),
    (wl.DTYPE_F32, 16, 4, 64, 8),
    (wl.DTYPE_BF16, 32, 4, 128, 64),
    (wl.DTYPE_BF16, 8, 8, 128, 1),
    (wl.DTYPE_BF16, 32, 8, 128, 256),
    (wl.DTYPE_F32, 4, 4, 128, 4),
    # groups of 16k heads: 16 query heads per warp on the MMA row side
    (wl.DTYPE_BF16, 64, 4, 128, 16),
    (wl.DTYPE_BF16, 64, 1, 128, 32),
    (wl.DTYPE_BF16, 64, 1, 64, 32),
    (wl.DTYPE_BF16, 128, 2, 128, 16),
    (wl.DTYPE_BF16, 64, 1, 128, 8),
    (wl.DTYPE_BF16, 256, 4, 128, 16),
    (wl.DTYPE_BF16, 32, 2, 128, 8),
]


@pytest.mark.parametrize("dtype,Hq,Hkv,D,bs", STREAM_SHAPES)
def test_stream_kernel_shapes(dtype, Hq, Hkv, D, bs):
    lens = [1, 15, 16, 17, 300, 1000, 2049, 4097]
    w = wl.custom_workload(dtype=dtype, batch=len(lens), num_q_heads=Hq, num_kv_heads=Hkv,
                           head_dim=D, block_size=bs, context_lens=lens, seed=Hq * 3 + bs,
                           new_tokens=True)
    d = upload(w)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gpu_write_and_decode(w, d, err)
    torch.cuda.synchronize()
    ref, _, _, _ = oracle_after_write(w)
    assert int(err.item()) == 0
    assert_close(to_f64(out), ref, dtype, f"stream {dtype} {Hq}/{Hkv} D{D} bs{bs}")


def test_stream_many_sequences_with_empty_ones():
    """700 sequences (more than one block of threads scans them), a third of
    them empty, in runs longer than a 32-wide window."""
    rng = np.random.default_rng(21)
    lens = rng.integers(1, 600, size=700)
    lens[rng.random(700) < 0.33] = 0
    lens[100:170] = 0  # a run of 70 empty sequences
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=700, num_q_heads=32, num_kv_heads=8,
                           head_dim=128, block_size=16, context_lens=lens.tolist(), seed=21,
                           new_tokens=True)
    d = upload(w)
    out = torch.full_like(d["q"], float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_write_kv_cache(d["key_cache"], d["value_cache"], d["k_new"], d["v_new"],
                         d["slot_mapping"], err_word=err)
    pa.pa_decode(out, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                 d["context_lens"], err_word=err)
    torch.cuda.synchronize()
    ref, _, _, _ = oracle_after_write(w)
    got = to_f64(out)
    assert int(err.item()) == 0
    assert np.all(got[lens == 0] == 0)
    assert_close(got, ref, w.dtype, "700 sequences")


@pytest.mark.parametrize("lens", [[100], [3, 5000], [1], [16, 16, 16]])
def test_stream_fewer_pages_than_ctas(lens):
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=len(lens), num_q_heads=32,
                           num_kv_heads=8, head_dim=128, block_size=16, context_lens=lens,
                           seed=len(lens), new_tokens=True)
    d = upload(w)
    out = gpu_write_and_decode(w, d)
    torch.cuda.synchronize()
    ref, _, _, _ = oracle_after_write(w)
    assert_close(to_f64(out), ref, w.dtype, f"lens {lens}")


def test_stream_repeated_calls_keep_workspace_clean():
    """Sequences split over many CTAs, decoded 5 times with the same
    workspace: identical bits every time (counters reset by the merging
    warp)."""
    w = wl.make_workload("long_bf16", seed=3, batch=2)
    d = upload(w)
    outs = []
    for _ in range(5):
        outs.append(gpu_write_and_decode(w, d).clone())
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o.view(torch.uint16), outs[0].view(torch.uint16))
    ref, _, _, _ = oracle_after_write(w)
    assert_close(to_f64(outs[0]), ref, w.dtype, "long split")


# Groups of 64 or 128 query heads per KV head decode on the tensor cores:
# 128-token tiles of every (sequence, KV head) pair split evenly over one CTA
# per SM; pairs cut between CTAs are merged by a second pass.
@pytest.mark.parametrize("Hq,Hkv,D,bs,lens", [
    (128, 2, 128, 16, [40000, 1, 0, 7000]),          # pairs spanning dozens of CTAs
    (64, 1, 128, 64, [129, 128, 127, 1, 2, 3, 4096]),
    (256, 2, 64, 32, [1000, 0, 33, 2500, 1]),         # 128 heads per KV head
])
def test_tensor_decode_long_and_ragged(Hq, Hkv, D, bs, lens):
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=len(lens), num_q_heads=Hq,
                           num_kv_heads=Hkv, head_dim=D, block_size=bs, context_lens=lens,
                           seed=Hq + bs, new_tokens=True)
    d = upload(w)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gpu_write_and_decode(w, d, err)
    again = torch.empty_like(out)
    pa.pa_decode(again, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                 d["context_lens"], err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref, _, _, _ = oracle_after_write(w)
    assert_close(to_f64(out), ref, w.dtype, f"tensor decode {Hq}/{Hkv} D{D} bs{bs}")
    assert torch.equal(out.view(torch.int16), again.view(torch.int16))
    for b, n in enumerate(lens):
        if n == 0:
            assert not to_f64(out)[b].any()


def test_tensor_decode_batch_above_one_scan_pass():
    """400 sequences of 64 query heads on one KV head: the tile kernel's
    prologue scans the context lengths in several passes of its threads."""
    rng = np.random.default_rng(12)
    lens = [int(x) for x in rng.integers(0, 300, size=400)]
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=len(lens), num_q_heads=64, num_kv_heads=1,
                           head_dim=128, block_size=32, context_lens=lens, seed=12,
                           new_tokens=True)
    d = upload(w)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gpu_write_and_decode(w, d, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref, _, _, _ = oracle_after_write(w)
    assert_close(to_f64(out), ref, w.dtype, "tensor decode, 400 sequences")
