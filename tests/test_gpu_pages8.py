"""8-token blocks on the page stream's tensor-copy path: a 16-token page is
two blocks of the table, each copied as its own boxes (serving page, section
5 on block sizes; teaching page, "Implementing teaching PagedAttention:
reading the historical KV cache from the block table").  Parity with the fp64
oracle through the C ABI: outputs within the bf16 tolerance, stored rows
bit-exact, bad ids in either block of a page flagged and zeroed."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_334_b200 import pa
from paged_kv_cache_334_b200 import workloads as wl

from _pa_helpers import assert_close, gpu_write_and_decode, oracle_after_write, to_f64, upload

pytestmark = pytest.mark.gpu

# lengths around the block (8) and page (16) edges, with the new token in the
# first and in the second block of its page, and long ragged ones
LENS = [1, 7, 8, 9, 15, 16, 17, 24, 25, 300, 1001, 2049, 4097]


def _forward(d, err):
    out = torch.empty_like(d["q"])
    pa.pa_forward_decode(out, d["q"], d["key_cache"], d["value_cache"], d["k_new"], d["v_new"],
                         d["slot_mapping"], d["block_tables"], d["context_lens"], err_word=err)
    return out


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (16, 4), (24, 8), (8, 8), (4, 4)])
@pytest.mark.parametrize("fused", [False, True])
def test_two_block_pages(Hq, Hkv, fused):
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=len(LENS), num_q_heads=Hq,
                           num_kv_heads=Hkv, head_dim=128, block_size=8, context_lens=LENS,
                           seed=Hq + 7 * Hkv, new_tokens=True)
    d = upload(w)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _forward(d, err) if fused else gpu_write_and_decode(w, d, err)
    torch.cuda.synchronize()
    ref, flags, kc, vc = oracle_after_write(w)
    assert int(err.item()) == 0 and not flags.any()
    assert_close(to_f64(out), ref, w.dtype, f"bs8 {Hq}/{Hkv} fused={fused}")
    # every stored row, bit for bit
    assert np.array_equal(d["key_cache"].view(torch.uint16).cpu().numpy(), kc)
    assert np.array_equal(d["value_cache"].view(torch.uint16).cpu().numpy(), vc)


def test_two_block_pages_bad_ids():
    """A bad id in the first or the second block of a visible page zeroes the
    sequence and sets the flag; an id past the last visible block (the
    second block of a page that ends in its first) is never read."""
    lens = [40, 40, 8, 300]
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=4, num_q_heads=32, num_kv_heads=8,
                           head_dim=128, block_size=8, context_lens=lens, seed=31,
                           max_blocks=40)
    bt = w.block_tables.copy()
    bt[0, 2] = w.num_blocks + 3   # first block of page 1 (tokens 16..23)
    bt[1, 3] = -1                 # second block of page 1 (tokens 24..31)
    bt[2, 1] = 987654321          # second block of page 0, past the 8 visible tokens
    d = upload(w)
    d["block_tables"] = torch.from_numpy(bt).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(d["q"])
    pa.pa_decode(out, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                 d["context_lens"], err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == pa.PA_DEVERR_BLOCK_ID
    ref, flags = oracle.decode(w.q, w.key_cache, w.value_cache, bt, w.context_lens)
    assert list(flags) == [oracle.FLAG_BLOCK_ID, oracle.FLAG_BLOCK_ID, 0, 0]
    got = to_f64(out)
    assert np.all(got[0] == 0) and np.all(got[1] == 0)
    assert_close(got, ref, w.dtype, "bs8 bad ids")


@pytest.mark.parametrize("P", [512, 32, 24])
def test_two_block_pages_splitk(P):
    """Split-K over 8-token blocks: partitions of whole 16-token pages run on
    the page stream, others (24 tokens) on the partition kernel; the merged
    result matches the oracle either way."""
    lens = [1, 9, 17, 100, 777, 2049]
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=len(lens), num_q_heads=32,
                           num_kv_heads=8, head_dim=128, block_size=8, context_lens=lens,
                           seed=P)
    d = upload(w)
    maxp = -(-w.max_blocks * w.block_size // P)
    pm = torch.empty(w.batch, 32, maxp, device="cuda")
    ps = torch.empty_like(pm)
    po = torch.empty(w.batch, 32, maxp, 128, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_decode_splitk(d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                        d["context_lens"], P, pm, ps, po, err_word=err)
    out = torch.empty_like(d["q"])
    pa.pa_reduce(out, pm, ps, po, d["context_lens"], P, err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref, flags = oracle.decode(w.q, w.key_cache, w.value_cache, w.block_tables, w.context_lens)
    assert not flags.any()
    assert_close(to_f64(out), ref, w.dtype, f"bs8 split-K P={P}")
