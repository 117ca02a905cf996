"""pa_decode_noalloc against pa_decode and the fp64 oracle, through the C ABI.

pa_decode_noalloc is the decode call for users of this library that may not
allocate device memory themselves -- for instance a plugin whose host engine
owns all device memory through its own pool, or a decode loop that cannot
afford the device-wide stalls cudaMalloc / cudaFree can cause -- and so
cannot pass pa_decode a workspace.  It uses a fixed scratch array inside the
library instead.  This file checks, on two calls in a row and on shapes that
alternate between calls (so leftovers of one call meet the next), that it
returns what pa_decode returns and what the oracle computes, within the
tolerances the other tests use; and, for a group of 64 query heads per KV
head (which pa_decode runs on its tensor-core tile kernel and
pa_decode_noalloc on the page-stream kernel), that it matches the oracle.

It is named to be collected last: a failure here does not hide any other
test when the run stops at the first failure.  It needs no state from other
tests and passes alone in a fresh process.
"""
import pytest
import torch

from paged_kv_cache_334_b200 import pa
from paged_kv_cache_334_b200 import workloads as wl

from _pa_helpers import assert_close, oracle_after_write, to_f64, upload

pytestmark = pytest.mark.gpu


def _prepare(w):
    d = upload(w)
    if "slot_mapping" in d:
        pa.pa_write_kv_cache(d["key_cache"], d["value_cache"], d["k_new"], d["v_new"],
                             d["slot_mapping"])
    ref = torch.empty_like(d["q"])
    pa.pa_decode(ref, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                 d["context_lens"])
    return d, ref


def _noalloc(d, err):
    out = torch.full_like(d["q"], float("nan"))
    pa.pa_decode_noalloc(out, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                         d["context_lens"], err_word=err)
    return out


def test_noalloc_matches_pa_decode_on_two_calls_in_a_row():
    w = wl.make_workload("gqa_bf16", seed=4)
    assert pa.pa_decode_workspace_bytes(upload_shape(w), w.batch, w.num_q_heads,
                                        w.max_blocks) <= pa.NOALLOC_SCRATCH_BYTES
    d, ref = _prepare(w)
    oref, flags, _, _ = oracle_after_write(w)
    assert not flags.any()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):
        out = _noalloc(d, err)
        torch.cuda.synchronize()
        assert_close(to_f64(out), to_f64(ref), w.dtype, f"noalloc call {call}")
        assert_close(to_f64(out), oref, w.dtype, f"noalloc call {call} vs oracle")
    assert int(err.item()) == 0


def test_noalloc_alternating_shapes_reuse_the_scratch():
    """Calls with different sizes share the scratch array; each one clears
    what it needs, so the previous call's leftovers do not leak in."""
    cases = [wl.make_workload("mixed_bf16", seed=1, batch=6),
             wl.make_workload("tiny_fp32", seed=0),
             wl.make_workload("gqa_bf16", seed=8, batch=12)]
    prepared = [(w, *_prepare(w), oracle_after_write(w)[0]) for w in cases]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for rnd in range(2):
        for w, d, ref, oref in prepared:
            out = _noalloc(d, err)
            torch.cuda.synchronize()
            assert_close(to_f64(out), to_f64(ref), w.dtype, f"{w.name} round {rnd}")
            assert_close(to_f64(out), oref, w.dtype, f"{w.name} round {rnd} vs oracle")
    assert int(err.item()) == 0


def test_noalloc_group_of_64_heads_on_the_page_stream():
    """64 query heads on one KV head: pa_decode takes the tensor-core tile
    path, pa_decode_noalloc the page-stream kernel (16 heads per consumer
    warp); both against the oracle, two calls in a row."""
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=6, num_q_heads=64, num_kv_heads=1,
                           head_dim=128, block_size=32, context_lens=[1, 31, 33, 700, 2100, 96],
                           seed=12, new_tokens=True)
    d, ref = _prepare(w)
    oref, flags, _, _ = oracle_after_write(w)
    assert not flags.any()
    assert_close(to_f64(ref), oref, w.dtype, "pa_decode, tensor-core path")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):
        out = _noalloc(d, err)
        torch.cuda.synchronize()
        assert_close(to_f64(out), oref, w.dtype, f"group of 64, call {call}")
    assert int(err.item()) == 0


def test_noalloc_eight_token_blocks():
    """8-token blocks, two to a page on the page stream: pa_decode_noalloc
    against pa_decode and the oracle, two calls in a row."""
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=7, num_q_heads=32, num_kv_heads=8,
                           head_dim=128, block_size=8, context_lens=[1, 8, 9, 16, 17, 300, 1025],
                           seed=13, new_tokens=True)
    d, ref = _prepare(w)
    oref, flags, _, _ = oracle_after_write(w)
    assert not flags.any()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):
        out = _noalloc(d, err)
        torch.cuda.synchronize()
        assert_close(to_f64(out), to_f64(ref), w.dtype, f"bs8 noalloc call {call}")
        assert_close(to_f64(out), oref, w.dtype, f"bs8 noalloc call {call} vs oracle")
    assert int(err.item()) == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # a table long enough for 65536 tokens per sequence: the workspace would
    # exceed the fixed scratch even though the actual contexts are short
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=64, num_q_heads=2, num_kv_heads=2,
                           head_dim=128, block_size=16, context_lens=[10] * 64, seed=2,
                           max_blocks=4096)
    need = pa.pa_decode_workspace_bytes(upload_shape(w), w.batch, w.num_q_heads, w.max_blocks)
    assert need > pa.NOALLOC_SCRATCH_BYTES
    d = upload(w)
    out = torch.zeros_like(d["q"])
    with pytest.raises(pa.PaError) as ei:
        pa.pa_decode_noalloc(out, d["q"], d["key_cache"], d["value_cache"],
                             d["block_tables"], d["context_lens"])
    assert ei.value.status == pa.PA_ERR_UNSUPPORTED
    assert "scratch" in str(ei.value)
    torch.cuda.synchronize()
    assert int(out.count_nonzero().item()) == 0  # nothing was enqueued


def upload_shape(w):
    """A stand-in with the cache's shape and dtype: the workspace size depends
    only on the cache descriptor, so no cache needs to be materialised."""
    dt = torch.float32 if w.dtype == wl.DTYPE_F32 else torch.bfloat16
    return torch.empty(1, 1, 1, 1, dtype=dt).expand(
        w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim)
