"""pa_decode_shared_prefix (suffix on the page-stream kernel, shared prefix on
tcgen05 tiles, merged in the prefix kernel's epilogue) against the fp64
oracle's decode of the same batch.

Tolerance: bf16, <= 2e-2 max-abs and <= 1e-2 mean-abs (as for pa_decode).
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


def shared_prefix(d, prefix_blocks, err=None):
    out = torch.empty_like(d["q"])
    pa.pa_decode_shared_prefix(out, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                               d["context_lens"], prefix_blocks, err_word=err)
    return out


def test_shared_prefix_mqa_workload():
    """The mqa_prefix_bf16 batch (256 sequences, 64 heads on 1 KV head, a
    2048-token shared prefix): the oracle's write + decode, and pa_decode."""
    w = wl.make_workload("mqa_prefix_bf16", seed=0)
    d = upload(w)
    pa.pa_write_kv_cache(d["key_cache"], d["value_cache"], d["k_new"], d["v_new"],
                         d["slot_mapping"])
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = shared_prefix(d, 2048 // w.block_size, err)
    ref_dec = torch.empty_like(d["q"])
    pa.pa_decode(ref_dec, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                 d["context_lens"])
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref, _, _, _ = oracle_after_write(w)
    assert_close(to_f64(out), ref, w.dtype, "shared prefix vs oracle")
    assert np.abs(to_f64(out) - to_f64(ref_dec)).max() <= 2e-2


PREFIX_CASES = [
    # Hq, Hkv, D, bs, prefix_blocks, suffix lengths
    (64, 1, 128, 32, 5, [1, 31, 32, 100, 700, 3]),        # partial last 128-row tile
    (64, 1, 64, 16, 9, [1, 16, 17, 300, 2]),              # head_dim 64; 144-token prefix
    # 8 heads per KV head, 4 KV heads: 16 sequences per tile, 17 sequences
    (32, 4, 128, 16, 8, [5, 77, 1, 128, 129, 40, 2, 9, 16, 17, 3, 300, 4, 60, 61, 1, 2]),
    (128, 1, 128, 32, 4, [1, 64, 65]),                    # 128 heads per KV head
    # 16 heads per KV head, 64-token pages: 8 sequences per tile, 9 sequences
    (64, 4, 128, 64, 3, [1, 200, 64, 63, 5, 6, 7, 129, 2]),
]


@pytest.mark.parametrize("Hq,Hkv,D,bs,npre,suffix", PREFIX_CASES)
def test_shared_prefix_shapes(Hq, Hkv, D, bs, npre, suffix):
    lens = [npre * bs + s for s in suffix]
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=len(lens), num_q_heads=Hq,
                           num_kv_heads=Hkv, head_dim=D, block_size=bs, context_lens=lens,
                           seed=Hq + D + bs + npre, prefix_blocks=npre, new_tokens=True)
    d = upload(w)
    pa.pa_write_kv_cache(d["key_cache"], d["value_cache"], d["k_new"], d["v_new"],
                         d["slot_mapping"])
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = shared_prefix(d, npre, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref, _, _, _ = oracle_after_write(w)
    assert_close(to_f64(out), ref, w.dtype, f"prefix {Hq}/{Hkv} D{D} bs{bs} P{npre}")


def test_shared_prefix_empty_suffix():
    """Sequences whose context is exactly the prefix."""
    npre, bs = 6, 32
    lens = [npre * bs, npre * bs + 1, npre * bs, npre * bs + 90]
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=len(lens), num_q_heads=64,
                           num_kv_heads=1, head_dim=128, block_size=bs, context_lens=lens,
                           seed=3, prefix_blocks=npre)
    d = upload(w)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = shared_prefix(d, npre, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref, _ = oracle.decode(w.q, w.key_cache, w.value_cache, w.block_tables, w.context_lens,
                           1.0 / math.sqrt(w.head_dim))
    assert_close(to_f64(out), ref, w.dtype, "empty suffix")


def test_shared_prefix_mismatch_is_flagged():
    """A table that leaves the prefix, and a context shorter than it: those
    sequences are flagged and zeroed, the others are unaffected."""
    npre, bs = 4, 32
    lens = [npre * bs + 50, npre * bs + 10, npre * bs + 7, npre * bs + 33]
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=len(lens), num_q_heads=64,
                           num_kv_heads=1, head_dim=128, block_size=bs, context_lens=lens,
                           seed=4, prefix_blocks=npre)
    d = upload(w)
    # sequence 1 reads another (valid) page in place of prefix page 2
    other = int(w.block_tables[0, npre])
    d["block_tables"][1, 2] = other
    # sequence 2 ends inside the prefix
    d["context_lens"][2] = npre * bs - 5
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = shared_prefix(d, npre, err)
    torch.cuda.synchronize()
    assert int(err.item()) & pa.PA_DEVERR_PREFIX
    got = to_f64(out)
    assert np.all(got[1] == 0) and np.all(got[2] == 0)
    ref, _ = oracle.decode(w.q, w.key_cache, w.value_cache, w.block_tables, w.context_lens,
                           1.0 / math.sqrt(w.head_dim))
    assert_close(got[[0, 3]], ref[[0, 3]], w.dtype, "unaffected sequences")


def test_shared_prefix_bad_block_zeroes_everything():
    npre, bs = 3, 32
    lens = [npre * bs + 5, npre * bs + 9]
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=2, num_q_heads=64, num_kv_heads=1,
                           head_dim=128, block_size=bs, context_lens=lens, seed=5,
                           prefix_blocks=npre)
    d = upload(w)
    d["block_tables"][:, 1] = w.num_blocks + 7  # the same bad id in every table
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = shared_prefix(d, npre, err)
    torch.cuda.synchronize()
    assert int(err.item()) & pa.PA_DEVERR_BLOCK_ID
    assert not to_f64(out).any()


def test_shared_prefix_zero_blocks_is_pa_decode():
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=3, num_q_heads=64, num_kv_heads=1,
                           head_dim=128, block_size=32, context_lens=[40, 1, 300], seed=6)
    d = upload(w)
    a = shared_prefix(d, 0)
    b = torch.empty_like(d["q"])
    pa.pa_decode(b, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                 d["context_lens"])
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


# Groups of 64 or 128 query heads per KV head take the tensor-core suffix
# kernel: 128-token tiles of each (sequence, KV head) pair split evenly over
# one CTA per SM, partials of pairs cut between CTAs folded in by the prefix
# kernel's epilogue.
TENSOR_SUFFIX_CASES = [
    # Hq, Hkv, D, bs, prefix_blocks, suffix lengths
    (64, 1, 128, 32, 2, [9000, 7000]),                      # pairs cut across many CTAs
    (128, 2, 128, 16, 4, [0, 300, 1, 128, 129, 2000, 5]),   # two KV heads, an empty suffix
    (64, 1, 128, 8, 16, [1, 127, 128, 129, 1000, 257]),     # 16 pages per tile
    (64, 1, 128, 128, 1, [1, 127, 128, 129, 600, 3]),       # one page per tile
    (256, 2, 64, 32, 3, [40, 700, 1, 0, 333]),              # 128 heads per KV head, head_dim 64
    (64, 1, 64, 16, 5, [2500, 2500, 2500, 1, 1, 1, 1, 1]),
]


def _decode_ref(w):
    return oracle.decode(w.q, w.key_cache, w.value_cache, w.block_tables, w.context_lens,
                         1.0 / math.sqrt(w.head_dim))[0]


@pytest.mark.parametrize("Hq,Hkv,D,bs,npre,suffix", TENSOR_SUFFIX_CASES)
def test_tensor_suffix_shapes(Hq, Hkv, D, bs, npre, suffix):
    lens = [npre * bs + s for s in suffix]
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=len(lens), num_q_heads=Hq,
                           num_kv_heads=Hkv, head_dim=D, block_size=bs, context_lens=lens,
                           seed=7 * Hq + D + bs + npre, prefix_blocks=npre)
    d = upload(w)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = shared_prefix(d, npre, err)
    again = shared_prefix(d, npre, err)  # the workspace is reused as is
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert_close(to_f64(out), _decode_ref(w), w.dtype, f"tensor suffix {Hq}/{Hkv} D{D} bs{bs}")
    assert torch.equal(out.view(torch.int16), again.view(torch.int16))


def test_tensor_suffix_bad_page_and_length():
    """A bad page id inside one suffix and a context longer than the table:
    those two sequences are flagged and zeroed, the others are unaffected."""
    npre, bs = 2, 32
    lens = [npre * bs + s for s in (900, 700, 50, 2000, 130)]
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=len(lens), num_q_heads=64,
                           num_kv_heads=1, head_dim=128, block_size=bs, context_lens=lens,
                           seed=11, prefix_blocks=npre)
    d = upload(w)
    d["block_tables"][1, npre + 5] = w.num_blocks + 3
    d["context_lens"][2] = w.block_tables.shape[1] * bs + 1
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = shared_prefix(d, npre, err)
    torch.cuda.synchronize()
    e = int(err.item())
    assert e & pa.PA_DEVERR_BLOCK_ID and e & pa.PA_DEVERR_CONTEXT_LEN
    got = to_f64(out)
    assert np.all(got[1] == 0) and np.all(got[2] == 0)
    ref = _decode_ref(w)
    keep = [0, 3, 4]
    assert_close(got[keep], ref[keep], w.dtype, "unaffected sequences")


def test_tensor_suffix_batch_above_one_scan_pass():
    """400 sequences: the suffix kernel's prologue takes several scan passes
    and the prefix kernel two waves of CTAs."""
    npre, bs = 3, 32
    rng = np.random.default_rng(13)
    lens = [npre * bs + int(x) for x in rng.integers(0, 200, size=400)]
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=len(lens), num_q_heads=64,
                           num_kv_heads=1, head_dim=128, block_size=bs, context_lens=lens,
                           seed=13, prefix_blocks=npre)
    d = upload(w)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = shared_prefix(d, npre, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert_close(to_f64(out), _decode_ref(w), w.dtype, "tensor suffix, 400 sequences")
