"""pa_forward_decode (one decode step: store each sequence's newest K/V row by
slot mapping, then decode) against the fp64 oracle's write + decode, and
against the two separate calls it replaces.

Tolerances as in the other parity tests: the stored rows bit-exact; the
attention output <= 1e-5 max-abs for fp32, <= 2e-2 max-abs and <= 1e-2
mean-abs for bf16.
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_334_b200 import pa
from paged_kv_cache_334_b200 import workloads as wl

from _pa_helpers import assert_close, oracle_after_write, to_dev, to_f64, upload

pytestmark = pytest.mark.gpu


def forward(d, err=None):
    out = torch.empty_like(d["q"])
    pa.pa_forward_decode(out, d["q"], d["key_cache"], d["value_cache"], d["k_new"], d["v_new"],
                         d["slot_mapping"], d["block_tables"], d["context_lens"], err_word=err)
    return out


def separate(d, err=None):
    pa.pa_write_kv_cache(d["key_cache"], d["value_cache"], d["k_new"], d["v_new"],
                         d["slot_mapping"], err_word=err)
    out = torch.empty_like(d["q"])
    pa.pa_decode(out, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                 d["context_lens"], err_word=err)
    return out


def rows_at(cache, slots, bs):
    s = torch.from_numpy(np.asarray(slots, dtype=np.int64)).cuda()
    return cache[s // bs, s % bs]


def raw(t):
    return t.view(torch.uint16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


def batch_rows(w):
    """New-token rows and slots indexed by sequence (the workloads list only
    the sequences with a non-empty context): empty sequences get a zero row
    and slot -1."""
    rows = np.flatnonzero(w.context_lens > 0)
    kn = np.zeros((w.batch,) + w.k_new.shape[1:], dtype=w.k_new.dtype)
    vn = np.zeros_like(kn)
    sm = np.full(w.batch, -1, dtype=np.int64)
    kn[rows], vn[rows], sm[rows] = w.k_new, w.v_new, w.slot_mapping
    return kn, vn, sm


def tiny_fp32_with_new_tokens():
    """The tiny fp32 shape (block size 4, 4 heads, head_dim 64) with each
    sequence's newest token written by the step."""
    return wl.custom_workload(dtype=wl.DTYPE_F32, batch=3, num_q_heads=4, num_kv_heads=4,
                              head_dim=64, block_size=4, context_lens=[5, 9, 12], seed=0,
                              new_tokens=True)


@pytest.mark.parametrize("name", ["tiny_fp32", "gqa_bf16", "mixed_bf16", "mqa_prefix_bf16"])
def test_forward_decode_workloads(name):
    """Output within tolerance of the oracle's write + decode; every stored
    row bit-exact; output bit-identical to pa_write_kv_cache + pa_decode."""
    w = tiny_fp32_with_new_tokens() if name == "tiny_fp32" else wl.make_workload(name, seed=0)
    assert (w.context_lens > 0).all() and w.slot_mapping.shape == (w.batch,)
    d = upload(w)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = forward(d, err)
    torch.cuda.synchronize()
    ref, flags, _, _ = oracle_after_write(w)
    assert not flags.any() and int(err.item()) == 0
    assert_close(to_f64(out), ref, w.dtype, name)
    got = rows_at(d["key_cache"], w.slot_mapping, w.block_size)
    assert raw(got).cpu().numpy().tobytes() == raw(d["k_new"]).cpu().numpy().tobytes()
    got = rows_at(d["value_cache"], w.slot_mapping, w.block_size)
    assert raw(got).cpu().numpy().tobytes() == raw(d["v_new"]).cpu().numpy().tobytes()
    # the same step as two calls, on a fresh copy of the caches
    d2 = upload(w)
    out2 = separate(d2)
    torch.cuda.synchronize()
    assert torch.equal(raw(out), raw(out2))
    assert torch.equal(raw(d["key_cache"]), raw(d2["key_cache"]))


def test_forward_decode_repeated_steps_are_identical():
    w = wl.make_workload("gqa_bf16", seed=3)
    d = upload(w)
    a = forward(d)
    b = forward(d)
    torch.cuda.synchronize()
    assert torch.equal(raw(a), raw(b))


def _slot_case(dtype, Hq, Hkv, D, bs):
    """Six sequences: 0 -> a slot that is not the table's (flagged, not stored,
    output zero); 1 -> slot -1 with its row already stored (nothing stored,
    normal output); 2 -> context 0 with a slot (flagged, output zero); 3..5
    normal, one of them a single token."""
    lens = [3 * bs + 5, 2 * bs, 0, 1, 5 * bs + 1, 700]
    w = wl.custom_workload(dtype=dtype, batch=len(lens), num_q_heads=Hq, num_kv_heads=Hkv,
                           head_dim=D, block_size=bs, context_lens=lens, seed=5,
                           new_tokens=True)
    kn, vn, sm = batch_rows(w)
    own0 = int(sm[0])
    used = set(int(x) for x in w.block_tables[w.block_tables >= 0].ravel())
    free = [b for b in range(w.num_blocks) if b not in used]
    assert free, "the pool needs a free block"
    bad_slot = free[0] * bs + 1
    sm[0] = bad_slot
    sm[1] = -1
    sm[2] = 7
    return w, kn, vn, sm, bad_slot, own0


@pytest.mark.parametrize("dtype,Hq,Hkv,D,bs", [
    (wl.DTYPE_BF16, 32, 8, 128, 16),   # persistent kernel, tensor-core consumers
    (wl.DTYPE_F32, 8, 4, 64, 8),       # persistent kernel, CUDA-core consumers
    (wl.DTYPE_BF16, 6, 2, 128, 16),    # group 3: partition kernel after a checked write
    (wl.DTYPE_BF16, 64, 1, 128, 32),   # group 64: tensor-core tiles after a checked write
    (wl.DTYPE_BF16, 128, 1, 64, 16),   # group 128, head_dim 64
])
def test_forward_decode_slot_checks(dtype, Hq, Hkv, D, bs):
    w, kn, vn, sm, bad_slot, own0 = _slot_case(dtype, Hq, Hkv, D, bs)
    d = upload(w)
    # sequence 1's newest row is already in the cache (an earlier write); the
    # workload lists the non-empty sequences 0, 1, 3, 4, 5, so it is row 1
    pa.pa_write_kv_cache(d["key_cache"], d["value_cache"], d["k_new"][1:2], d["v_new"][1:2],
                         d["slot_mapping"][1:2])
    before_bad = rows_at(d["key_cache"], [bad_slot], bs).clone()
    d["k_new"], d["v_new"] = to_dev(kn, w.dtype), to_dev(vn, w.dtype)
    d["slot_mapping"] = torch.from_numpy(sm).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = forward(d, err)
    torch.cuda.synchronize()
    assert int(err.item()) == pa.PA_DEVERR_SLOT
    got = to_f64(out)
    assert np.all(got[0] == 0) and np.all(got[2] == 0)
    # nothing stored at the rejected slot, nor at sequence 0's own slot
    assert torch.equal(raw(rows_at(d["key_cache"], [bad_slot], bs)), raw(before_bad))
    own = rows_at(d["key_cache"], [own0], bs)
    assert torch.isnan(own.float()).all()
    # the other sequences match the oracle's write (of sequences 1 and 3..5) + decode
    ref, _, _, _ = oracle_after_write(w)
    keep = [1, 3, 4, 5]
    assert_close(got[keep], ref[keep], w.dtype, "valid sequences")


def test_forward_decode_empty_batch_is_a_no_op():
    kc = torch.zeros(4, 16, 8, 128, dtype=torch.bfloat16, device="cuda")
    q = torch.zeros(0, 32, 128, dtype=torch.bfloat16, device="cuda")
    e = torch.zeros(0, 8, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    pa.pa_forward_decode(out, q, kc, kc.clone(), e, e, torch.zeros(0, dtype=torch.int64,
                                                                   device="cuda"),
                         torch.zeros(0, 4, dtype=torch.int32, device="cuda"),
                         torch.zeros(0, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
