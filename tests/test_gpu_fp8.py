"""FP8 (E4M3) KV pages through the C ABI against the fp64 oracle.

The write (bf16 rows divided by the tensor's scale in IEEE single precision,
rounded to the nearest E4M3 code, saturating at 448) is bit-exact; decode
over the pages (values code * scale, q bf16) is held to the bf16 tolerance
(<= 2e-2 max-abs, <= 1e-2 mean-abs): the kernel converts the codes exactly
to fp16 and computes in fp16 tiles with fp32 accumulation.  Unused slots hold the NaN code 0x7F, so an
over-read shows as NaN.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_334_b200 import pa
from paged_kv_cache_334_b200 import workloads as wl

from _pa_helpers import assert_close, to_f64

pytestmark = pytest.mark.gpu


def up(a: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if a.dtype == np.uint8:
        t = t.view(torch.float8_e4m3fn)
    elif a.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t.cuda()


def codes(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.uint8).cpu().numpy()


def bf16_bits(x) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.uint16).numpy().copy()


@pytest.mark.parametrize("k_scale,v_scale", [(0.25, 2.0), (0.3, 0.0117)])
def test_fp8_write_is_bit_exact(k_scale, v_scale):
    NB, bs, Hkv, D, N = 40, 16, 8, 128, 37
    rng = np.random.default_rng(int(k_scale * 1000))
    vals = rng.normal(0, 3, size=(N, Hkv, D)).astype(np.float32)
    # ties between neighbouring codes (exact after division by a power of two),
    # saturation, signed zero, subnormal codes
    pos = oracle.e4m3_value(np.arange(0x7F, dtype=np.uint8))
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)
    special = np.concatenate([mids, -mids, [0.0, -0.0, 600.0, -1e4, 2.0 ** -12]]).astype(np.float32)
    flat = vals.reshape(-1)
    flat[:special.size] = special * np.float32(k_scale)
    k_new = bf16_bits(vals)
    v_new = bf16_bits(rng.normal(0, 0.05, size=(N, Hkv, D)))
    slots = rng.choice(NB * bs, size=N, replace=False).astype(np.int64)
    slots[3] = -1
    kc = np.full((NB, bs, Hkv, D), 0x7F, dtype=np.uint8)
    vc = kc.copy()
    dk, dv = up(kc), up(vc)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_write_kv_cache(dk, dv, up(k_new), up(v_new), torch.from_numpy(slots).cuda(),
                         err_word=err, k_scale=k_scale, v_scale=v_scale)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert oracle.write_kv_cache_fp8(kc, vc, k_new, v_new, slots, k_scale, v_scale) == 0
    assert np.array_equal(codes(dk), kc)
    assert np.array_equal(codes(dv), vc)


def _oracle_step(w):
    kc, vc = w.key_cache.copy(), w.value_cache.copy()
    assert oracle.write_kv_cache_fp8(kc, vc, w.k_new, w.v_new, w.slot_mapping, w.k_scale,
                                     w.v_scale) == 0
    ref, _ = oracle.decode_fp8(w.q, kc, vc, w.k_scale, w.v_scale, w.block_tables,
                               w.context_lens, 1.0 / math.sqrt(w.head_dim))
    return ref


def _upload(w):
    return dict(q=up(w.q), kc=up(w.key_cache), vc=up(w.value_cache), kn=up(w.k_new),
                vn=up(w.v_new), sm=torch.from_numpy(w.slot_mapping).cuda(),
                bt=torch.from_numpy(w.block_tables).cuda(),
                cl=torch.from_numpy(w.context_lens).cuda())


def test_fp8_gqa_workload_write_then_decode_and_forward():
    w = wl.make_workload("gqa_fp8", seed=0)
    ref = _oracle_step(w)
    d = _upload(w)
    sc = dict(k_scale=w.k_scale, v_scale=w.v_scale)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    # two calls: the write, then the decode
    pa.pa_write_kv_cache(d["kc"], d["vc"], d["kn"], d["vn"], d["sm"], err_word=err, **sc)
    out = torch.empty_like(d["q"])
    pa.pa_decode(out, d["q"], d["kc"], d["vc"], d["bt"], d["cl"], err_word=err, **sc)
    # one call: the fused step on a fresh copy of the pages
    d2 = _upload(w)
    out2 = torch.empty_like(d2["q"])
    pa.pa_forward_decode(out2, d2["q"], d2["kc"], d2["vc"], d2["kn"], d2["vn"], d2["sm"],
                         d2["bt"], d2["cl"], err_word=err, **sc)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert_close(to_f64(out), ref, wl.DTYPE_BF16, "fp8 write + decode")
    assert_close(to_f64(out2), ref, wl.DTYPE_BF16, "fp8 forward decode")
    # the fused write stored the same codes as the separate one
    assert torch.equal(d["kc"].view(torch.uint8), d2["kc"].view(torch.uint8))
    assert torch.equal(d["vc"].view(torch.uint8), d2["vc"].view(torch.uint8))


FP8_SHAPES = [
    # Hq, Hkv, bs
    (32, 8, 16),   # 4 query heads per KV head
    (8, 8, 16),    # 1
    (16, 4, 16),   # 16-token blocks two to a page at 4 KV heads
    (32, 4, 16),   # 8
    (16, 8, 256),  # 256-token pages in 32-token virtual pages
    (16, 4, 32),
    (8, 4, 64),    # 2
    (32, 4, 128),  # 8
]


@pytest.mark.parametrize("Hq,Hkv,bs", FP8_SHAPES)
def test_fp8_shapes(Hq, Hkv, bs):
    # around the 16-token tiles and the 32-token pages (the new token in
    # either block of a two-block page)
    lens = [1, 15, 16, 17, 31, 32, 33, 48, 49, 300, 1000, 2049]
    w = wl.custom_workload(dtype=wl.DTYPE_FP8, batch=len(lens), num_q_heads=Hq,
                           num_kv_heads=Hkv, head_dim=128, block_size=bs, context_lens=lens,
                           seed=Hq + Hkv + bs, new_tokens=True, k_scale=0.125, v_scale=0.75)
    ref = _oracle_step(w)
    d = _upload(w)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(d["q"])
    pa.pa_forward_decode(out, d["q"], d["kc"], d["vc"], d["kn"], d["vn"], d["sm"], d["bt"],
                         d["cl"], err_word=err, k_scale=w.k_scale, v_scale=w.v_scale)
    noa = torch.empty_like(out)
    pa.pa_decode_noalloc(noa, d["q"], d["kc"], d["vc"], d["bt"], d["cl"], err_word=err,
                         k_scale=w.k_scale, v_scale=w.v_scale)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert_close(to_f64(out), ref, wl.DTYPE_BF16, f"fp8 {Hq}/{Hkv} bs{bs}")
    assert torch.equal(out.view(torch.int16), noa.view(torch.int16))


def test_fp8_forward_bad_slot_is_flagged_and_zeroed():
    lens = [40, 17, 300]
    w = wl.custom_workload(dtype=wl.DTYPE_FP8, batch=3, num_q_heads=32, num_kv_heads=8,
                           head_dim=128, block_size=16, context_lens=lens, seed=9,
                           new_tokens=True)
    ref = _oracle_step(w)
    d = _upload(w)
    used = set(int(x) for x in w.block_tables[w.block_tables >= 0].ravel())
    free = [b for b in range(w.num_blocks) if b not in used]
    d["sm"][1] = free[0] * 16 + 3  # not the slot the table gives position 16
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(d["q"])
    pa.pa_forward_decode(out, d["q"], d["kc"], d["vc"], d["kn"], d["vn"], d["sm"], d["bt"],
                         d["cl"], err_word=err, k_scale=w.k_scale, v_scale=w.v_scale)
    torch.cuda.synchronize()
    assert int(err.item()) == pa.PA_DEVERR_SLOT
    got = to_f64(out)
    assert not got[1].any()
    assert_close(got[[0, 2]], ref[[0, 2]], wl.DTYPE_BF16, "unaffected sequences")


def test_fp8_bad_ids_in_either_block_of_a_page():
    """16-token blocks go two to a 32-token page: a bad id in the first or
    the second block of a visible page zeroes the sequence and sets the flag;
    the second entry of a page that ends in its first block is never read."""
    lens = [40, 40, 16, 300]
    w = wl.custom_workload(dtype=wl.DTYPE_FP8, batch=4, num_q_heads=32, num_kv_heads=8,
                           head_dim=128, block_size=16, context_lens=lens, seed=41,
                           max_blocks=24)
    bt = w.block_tables.copy()
    bt[0, 1] = w.num_blocks + 2   # second block of page 0 (tokens 16..31)
    bt[1, 2] = -5                 # first block of page 1 (tokens 32..47)
    bt[2, 1] = 123456789          # past the 16 visible tokens: never read
    d = dict(q=up(w.q), kc=up(w.key_cache), vc=up(w.value_cache),
             bt=torch.from_numpy(bt).cuda(), cl=torch.from_numpy(w.context_lens).cuda())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(d["q"])
    pa.pa_decode(out, d["q"], d["kc"], d["vc"], d["bt"], d["cl"], err_word=err,
                 k_scale=w.k_scale, v_scale=w.v_scale)
    torch.cuda.synchronize()
    assert int(err.item()) == pa.PA_DEVERR_BLOCK_ID
    ref, flags = oracle.decode_fp8(w.q, w.key_cache, w.value_cache, w.k_scale, w.v_scale, bt,
                                   w.context_lens, 1.0 / math.sqrt(w.head_dim))
    assert list(flags) == [oracle.FLAG_BLOCK_ID, oracle.FLAG_BLOCK_ID, 0, 0]
    got = to_f64(out)
    assert not got[0].any() and not got[1].any()
    assert_close(got, ref, wl.DTYPE_BF16, "fp8 bad ids")


def test_fp8_unsupported_shapes_are_refused():
    q = torch.zeros(2, 32, 128, dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros(2, 4, dtype=torch.int32, device="cuda")
    cl = torch.ones(2, dtype=torch.int32, device="cuda")

    def cache(nb, bs, hkv, d):
        return torch.zeros(nb, bs, hkv, d, dtype=torch.uint8, device="cuda").view(
            torch.float8_e4m3fn)

    big = torch.zeros(2, 64, 128, dtype=torch.bfloat16, device="cuda")
    for kc, qq in [(cache(8, 8, 8, 128), q),                 # 8-token pages
                   (cache(8, 16, 16, 128), q),               # 16 KV heads (group 2)
                   (cache(8, 16, 2, 128), q),                # 2 KV heads (group 16)
                   (cache(8, 16, 4, 128), big)]:             # group 16
        out = torch.empty_like(qq)
        with pytest.raises(pa.PaError) as e:
            pa.pa_decode(out, qq, kc, kc.clone(), bt, cl, k_scale=1.0, v_scale=1.0)
        assert e.value.status == pa.PA_ERR_UNSUPPORTED
    kc = cache(8, 16, 8, 64)
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode(torch.empty(2, 32, 64, dtype=torch.bfloat16, device="cuda"),
                     torch.zeros(2, 32, 64, dtype=torch.bfloat16, device="cuda"), kc, kc.clone(),
                     bt, cl)
    assert e.value.status == pa.PA_ERR_UNSUPPORTED
    kc = cache(8, 16, 8, 128)
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode(torch.empty_like(q), q, kc, kc.clone(), bt, cl, k_scale=0.0)
    assert e.value.status == pa.PA_ERR_INVALID_ARG
