"""The C ABI library on a machine without a GPU: it loads, exports every
symbol include/pa.h declares, and its host-side argument checks return the
documented statuses before any device work (no compute calls here)."""
import ctypes
import os
import re

import pytest

from paged_kv_cache_334_b200 import pa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", fn)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        names |= set(re.findall(r"\b(pa_\w+)\s*\(", src))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_334_b200 import build
    build.build()
    return pa.load()


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("pa_write_kv_cache", "pa_decode", "pa_decode_splitk", "pa_reduce"):
        assert required in names
    assert set(pa.EXPORTED_SYMBOLS) <= set(names)


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, f"not exported: {missing}"


def test_version_and_status_strings(lib):
    assert pa.pa_version() >= 100
    assert lib.pa_status_string(0) == b"PA_OK"
    assert lib.pa_status_string(1) == b"PA_ERR_INVALID_ARG"
    assert lib.pa_status_string(2) == b"PA_ERR_UNSUPPORTED"
    assert lib.pa_status_string(3) == b"PA_ERR_CUDA"


def _desc(nb=16, bs=16, hkv=8, d=128, dtype=1):
    return pa.CacheDesc(nb, bs, hkv, d, dtype)


FAKE = ctypes.c_void_p(0x10000)       # aligned, never dereferenced
MISALIGNED = ctypes.c_void_p(0x10008)


def _decode(lib, desc, *, out=FAKE, q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, cl=FAKE, B=2, Hq=32,
            MB=4, scale=0.1, ws=FAKE, wsb=1 << 30):
    return lib.pa_decode(ctypes.byref(desc) if desc is not None else None, out, q, kc, vc, bt,
                         cl, B, Hq, MB, scale, ws, wsb, None, None)


def test_decode_argument_checks(lib):
    assert _decode(lib, None) == pa.PA_ERR_INVALID_ARG
    assert _decode(lib, _desc(d=96)) == pa.PA_ERR_UNSUPPORTED
    assert _decode(lib, _desc(bs=12)) == pa.PA_ERR_UNSUPPORTED
    assert _decode(lib, _desc(bs=512)) == pa.PA_ERR_UNSUPPORTED
    assert _decode(lib, _desc(dtype=7)) == pa.PA_ERR_INVALID_ARG
    assert _decode(lib, _desc(), Hq=30) == pa.PA_ERR_INVALID_ARG       # not a multiple of Hkv
    assert _decode(lib, _desc(), B=-1) == pa.PA_ERR_INVALID_ARG
    assert _decode(lib, _desc(), q=MISALIGNED) == pa.PA_ERR_INVALID_ARG
    assert _decode(lib, _desc(), kc=None) == pa.PA_ERR_INVALID_ARG
    assert _decode(lib, _desc(), cl=None) == pa.PA_ERR_INVALID_ARG
    assert _decode(lib, _desc(), scale=float("inf")) == pa.PA_ERR_INVALID_ARG
    assert _decode(lib, _desc(), wsb=16) == pa.PA_ERR_INVALID_ARG       # workspace too small
    assert _decode(lib, _desc(), ws=ctypes.c_void_p(0x10010)) == pa.PA_ERR_INVALID_ARG
    assert _decode(lib, _desc(hkv=1), Hq=1024) == pa.PA_ERR_UNSUPPORTED  # group > 512
    assert b"head_dim" in _msg(lib, _decode(lib, _desc(d=96)))
    # an empty batch is a valid no-op (no device work)
    assert _decode(lib, _desc(), B=0) == pa.PA_OK


def _msg(lib, _status):
    return lib.pa_last_error_message()


def test_splitk_and_reduce_argument_checks(lib):
    d = _desc()
    f = lib.pa_decode_splitk
    # partition not a multiple of the block size
    assert f(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 2, 32, 4, 0.1, 24, 8, FAKE, FAKE,
             FAKE, None, None) == pa.PA_ERR_INVALID_ARG
    # too few partitions for max_blocks * block_size tokens
    assert f(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 2, 32, 64, 0.1, 256, 3, FAKE, FAKE,
             FAKE, None, None) == pa.PA_ERR_INVALID_ARG
    # more than 1024 blocks in one partition, on a shape only the partition
    # kernel serves (fp32 pages with 2 KV heads; the page-stream kernel has no
    # such limit)
    assert f(ctypes.byref(_desc(bs=1, hkv=2, dtype=0)), FAKE, FAKE, FAKE, FAKE, FAKE, 2, 32, 4096,
             0.1, 2048, 2, FAKE, FAKE, FAKE, None, None) == pa.PA_ERR_UNSUPPORTED
    r = lib.pa_reduce
    assert r(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 32, 128, 512, 4, 9, None, None) == pa.PA_ERR_INVALID_ARG
    assert r(MISALIGNED, FAKE, FAKE, FAKE, FAKE, 2, 32, 128, 512, 4, 1, None, None) == \
        pa.PA_ERR_INVALID_ARG
    assert r(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 32, 128, 512, 4, 1, None, None) == pa.PA_OK


def test_write_argument_checks(lib):
    d = _desc()
    w = lib.pa_write_kv_cache
    assert w(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, -1, None, None) == pa.PA_ERR_INVALID_ARG
    assert w(ctypes.byref(d), FAKE, FAKE, MISALIGNED, FAKE, FAKE, 3, None, None) == \
        pa.PA_ERR_INVALID_ARG
    assert w(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, None, 3, None, None) == pa.PA_ERR_INVALID_ARG
    assert w(ctypes.byref(d), None, None, None, None, None, 0, None, None) == pa.PA_OK


def test_workspace_size(lib):
    d = _desc(nb=100, bs=16, hkv=8, d=128)
    n = lib.pa_decode_workspace_bytes(ctypes.byref(d), 32, 32, 128)
    assert n > 0 and n % 256 == 0
    # partial max, sum and output per (sequence, query head, 256-token partition)
    parts = (128 * 16 + 255) // 256
    assert n >= 32 * 32 * parts * (2 + 128) * 4
    assert lib.pa_decode_workspace_bytes(ctypes.byref(d), 32, 30, 128) == 0
    assert lib.pa_decode_workspace_bytes(None, 32, 32, 128) == 0


def test_noalloc_size_limit_and_argument_checks(lib):
    """pa_decode_noalloc refuses sizes whose workspace exceeds its fixed
    scratch before any device work, and passes other argument errors
    through from pa_decode."""
    d = _desc(nb=100000, bs=16, hkv=2, d=128)
    need = lib.pa_decode_workspace_bytes(ctypes.byref(d), 4096, 2, 1024)
    assert need > pa.NOALLOC_SCRATCH_BYTES
    f = lib.pa_decode_noalloc
    assert f(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4096, 2, 1024, 0.1, None,
             None) == pa.PA_ERR_UNSUPPORTED
    assert b"scratch" in lib.pa_last_error_message()
    assert f(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 32, 4, 0.1, None, None) == \
        pa.PA_ERR_INVALID_ARG
    assert f(ctypes.byref(_desc(d=96)), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 32, 4, 0.1, None,
             None) == pa.PA_ERR_UNSUPPORTED
    assert f(ctypes.byref(_desc()), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 32, 4, 0.1, None,
             None) == pa.PA_OK


def test_forward_decode_argument_checks(lib):
    """pa_forward_decode: the slot mapping and the new rows are required and
    checked before any device work; the rest are pa_decode's checks."""
    f = lib.pa_forward_decode
    d = _desc()

    def call(k_new=FAKE, v_new=FAKE, sm=FAKE, B=2, Hq=32, dsc=d):
        return f(ctypes.byref(dsc), FAKE, FAKE, FAKE, FAKE, k_new, v_new, sm, FAKE, FAKE, B, Hq,
                 4, 0.1, FAKE, 1 << 30, None, None)

    assert call(sm=None) == pa.PA_ERR_INVALID_ARG
    assert b"slot_mapping" in lib.pa_last_error_message()
    assert call(k_new=None) == pa.PA_ERR_INVALID_ARG
    assert call(v_new=MISALIGNED) == pa.PA_ERR_INVALID_ARG
    assert call(Hq=30) == pa.PA_ERR_INVALID_ARG
    assert call(dsc=_desc(d=96)) == pa.PA_ERR_UNSUPPORTED
    assert call(B=0, sm=None, k_new=None, v_new=None) == pa.PA_OK


def _fp8(nb=16, bs=16, hkv=8, d=128, ks=0.25, vs=0.5):
    return pa.CacheDesc(nb, bs, hkv, d, pa.PA_DTYPE_FP8_E4M3, ks, vs)


def test_fp8_argument_checks_need_no_device(lib):
    """FP8 pages: scales and shapes are checked on the host, before any
    device work (every pointer here is fake)."""
    # scales must be finite and > 0
    for ks, vs in [(0.0, 1.0), (1.0, -1.0), (float("nan"), 1.0), (float("inf"), 1.0)]:
        assert _decode(lib, _fp8(ks=ks, vs=vs)) == pa.PA_ERR_INVALID_ARG
    assert b"scales" in lib.pa_last_error_message()
    # head_dim 128 only
    assert _decode(lib, _fp8(d=64)) == pa.PA_ERR_UNSUPPORTED
    # the page-stream shapes: block_size >= 16, 4 or 8 KV heads, <= 8 heads per KV head
    assert _decode(lib, _fp8(bs=8)) == pa.PA_ERR_UNSUPPORTED
    assert _decode(lib, _fp8(hkv=2), Hq=4) == pa.PA_ERR_UNSUPPORTED
    assert _decode(lib, _fp8(hkv=4), Hq=64) == pa.PA_ERR_UNSUPPORTED
    assert b"FP8" in lib.pa_last_error_message()
    # split-K partials of FP8 pages: the page-stream shapes only; the
    # shared-prefix call takes bf16 pages only
    P = 8
    assert lib.pa_decode_splitk(ctypes.byref(_fp8(hkv=2)), FAKE, FAKE, FAKE, FAKE, FAKE, 2, 4, 4,
                                0.1, 16, P, FAKE, FAKE, FAKE, None, None) == pa.PA_ERR_UNSUPPORTED
    assert b"FP8" in lib.pa_last_error_message()
    # FP8 pages stream 32 tokens at a time: partitions must hold whole pages
    assert lib.pa_decode_splitk(ctypes.byref(_fp8()), FAKE, FAKE, FAKE, FAKE, FAKE, 2, 32, 4,
                                0.1, 16, P, FAKE, FAKE, FAKE, None, None) == pa.PA_ERR_UNSUPPORTED
    assert lib.pa_decode_shared_prefix(ctypes.byref(_fp8()), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                       2, 32, 4, 1, 0.1, FAKE, 1 << 30, None,
                                       None) == pa.PA_ERR_UNSUPPORTED
    # the write: the same descriptor checks
    assert lib.pa_write_kv_cache(ctypes.byref(_fp8(d=64)), FAKE, FAKE, FAKE, FAKE, FAKE, 2, None,
                                 None) == pa.PA_ERR_UNSUPPORTED
    assert lib.pa_write_kv_cache(ctypes.byref(_fp8(ks=0.0)), FAKE, FAKE, FAKE, FAKE, FAKE, 2,
                                 None, None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_version() == 300


def _round256(x):
    return (x + 255) // 256 * 256


def test_workspace_sizes_of_the_tensor_core_path(lib):
    """Groups of 64 or 128 query heads (bf16) decode on the tile kernel: the
    workspace holds per-CTA partials for 192 CTAs x 2 slots, one 16-byte
    record per (sequence, KV head) and each row's fp32 result, independent
    of the table width; the shared-prefix call asks for at least as much."""
    for hkv, hq, d in [(1, 64, 128), (2, 128, 128), (1, 128, 64)]:
        desc = _desc(nb=1000, bs=32, hkv=hkv, d=d)
        B = 300
        slots = 192 * 2 * hq
        rows = B * hq
        want = _round256(slots * 2 * 4)
        want = _round256(want + slots * d * 4)
        want = _round256(want + B * hkv * 16)
        want = _round256(want + rows * 2 * 4)
        want = _round256(want + rows * d * 4)
        for mb in (4, 500):
            got = lib.pa_decode_workspace_bytes(ctypes.byref(desc), B, hq, mb)
            assert got == want, (hkv, hq, d, mb, got, want)
        assert lib.pa_decode_shared_prefix_workspace_bytes(ctypes.byref(desc), B, hq, 500,
                                                           64) >= want
    # a group of 32 stays on the page stream: partials for 192 CTAs x 2
    # slots plus 16 bytes of counters per sequence, so the batch adds only
    # the counters
    desc = _desc(nb=1000, bs=32, hkv=2, d=128)
    one = lib.pa_decode_workspace_bytes(ctypes.byref(desc), 1, 64, 500)
    many = lib.pa_decode_workspace_bytes(ctypes.byref(desc), 300, 64, 500)
    assert one >= 192 * 2 * 64 * 128 * 4
    assert 0 <= many - one <= _round256(300 * 16)


def test_noalloc_refuses_what_its_scratch_cannot_hold(lib):
    """pa_decode_noalloc uses the page-stream layout in its 16 MiB scratch and
    refuses, before touching the device, sizes whose layout is larger."""
    f = lib.pa_decode_noalloc
    desc = _desc(nb=1000, bs=32, hkv=1, d=128)
    # 128 query heads: the partials alone take 192 x 2 x 128 x 128 x 4 bytes
    assert f(ctypes.byref(desc), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 128, 4096, 0.1,
             None, None) == pa.PA_ERR_UNSUPPORTED
    assert b"scratch" in lib.pa_last_error_message()
    # the partition kernel's workspace grows with batch x partitions: fp32
    # pages with 2 KV heads (a shape the page-stream kernel does not serve),
    # 8 sequences of up to 131072 tokens need 512 partials per row
    fp32 = _desc(nb=1000, bs=32, hkv=2, d=128, dtype=0)
    assert f(ctypes.byref(fp32), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 8, 32, 4096, 0.1,
             None, None) == pa.PA_ERR_UNSUPPORTED
    assert b"scratch" in lib.pa_last_error_message()


def test_prefill_argument_checks(lib):
    """pa_prefill refuses, before touching the device, what its tensor-core
    tiles cannot serve, and does nothing for empty work."""
    f = lib.pa_prefill

    def call(desc, *, out=FAKE, q=FAKE, qs=FAKE, B=2, T=64, Hq=32, MB=16, mql=32, scale=0.1):
        return f(ctypes.byref(desc), out, q, FAKE, FAKE, FAKE, FAKE, qs, B, T, Hq, MB, mql,
                 scale, None, None)

    bf = _desc(nb=64, bs=16, hkv=8, d=128)
    assert call(_desc(nb=64, bs=16, hkv=8, d=128, dtype=0)) == pa.PA_ERR_UNSUPPORTED  # fp32
    assert b"bf16" in lib.pa_last_error_message()
    assert call(_fp8()) == pa.PA_ERR_UNSUPPORTED
    assert call(bf, Hq=24) == pa.PA_ERR_UNSUPPORTED        # 3 heads per KV head
    assert call(_desc(nb=64, bs=256, hkv=1, d=128), Hq=256) == pa.PA_ERR_UNSUPPORTED
    assert call(_desc(nb=64, bs=4, hkv=8, d=128)) == pa.PA_ERR_UNSUPPORTED
    assert call(bf, MB=4097) == pa.PA_ERR_UNSUPPORTED       # table slice past shared memory
    assert call(bf, Hq=20) == pa.PA_ERR_INVALID_ARG         # not a multiple of Hkv
    assert call(bf, T=-1) == pa.PA_ERR_INVALID_ARG
    assert call(bf, mql=-1) == pa.PA_ERR_INVALID_ARG
    assert call(bf, B=70000) == pa.PA_ERR_INVALID_ARG
    assert call(bf, scale=float("nan")) == pa.PA_ERR_INVALID_ARG
    assert call(bf, q=MISALIGNED) == pa.PA_ERR_INVALID_ARG
    assert call(bf, out=None) == pa.PA_ERR_INVALID_ARG
    assert call(bf, qs=None) == pa.PA_ERR_INVALID_ARG
    # empty work: nothing to launch
    assert call(bf, B=0) == pa.PA_OK
    assert call(bf, T=0) == pa.PA_OK
    assert call(bf, mql=0) == pa.PA_OK
