"""fp64 CPU oracle for paged decode attention -- TEST INFRASTRUCTURE ONLY.

Only the tests, the package's smoke check and the benchmark's CPU-baseline
leg may import this package.  The product path never does: it has no CPU
fallback.  The arithmetic lives in ``pa_oracle.c`` (plain C, double
precision, OpenMP over query heads), built with gcc by :func:`build`; this
module only marshals numpy arrays into it.

Each function cites the passage it follows in its docstring; the C source
restates them in full.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB = os.path.join(_HERE, "libpa_oracle.so")

FLAG_BLOCK_ID = 1
FLAG_CONTEXT_LEN = 2
FLAG_SLOT = 4

_lib = None


def build(force: bool = False) -> str:
    """Compile pa_oracle.c into libpa_oracle.so next to it (gcc, -O2, OpenMP,
    no fast-math, no FMA contraction so double rounding stays textbook)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
               "-ffp-contract=off", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32, i64, dbl = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        lib.orc_set_num_threads.argtypes = [ctypes.c_int]
        lib.orc_set_num_threads.restype = None
        lib.orc_max_threads.argtypes = []
        lib.orc_max_threads.restype = ctypes.c_int
        lib.orc_map_token.argtypes = [P, i32, i32, i32, i64, P, P]
        lib.orc_map_token.restype = ctypes.c_int
        lib.orc_widen.argtypes = [P, ctypes.c_int, i64, P]
        lib.orc_widen.restype = None
        lib.orc_gather_kv.argtypes = [P, P, ctypes.c_int, i32, i32, i32, i32, P, i32, i32, P, P]
        lib.orc_gather_kv.restype = ctypes.c_int
        lib.orc_attention.argtypes = [P, P, P, i32, i32, i32, i32, dbl, P]
        lib.orc_attention.restype = None
        lib.orc_decode.argtypes = [P, P, P, ctypes.c_int, i32, i32, i32, i32, P, P, i32, i32,
                                   i32, dbl, P, P]
        lib.orc_decode.restype = ctypes.c_int
        lib.orc_partials.argtypes = [P, P, P, ctypes.c_int, i32, i32, i32, i32, P, P, i32, i32,
                                     i32, dbl, i32, i32, P, P, P]
        lib.orc_partials.restype = ctypes.c_int
        lib.orc_merge.argtypes = [P, P, P, i32, i32, i32, i32, P]
        lib.orc_merge.restype = None
        lib.orc_write_kv_cache.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32]
        lib.orc_write_kv_cache.restype = ctypes.c_int
        f32 = ctypes.c_float
        lib.orc_prefill.argtypes = [P, P, P, ctypes.c_int, i32, i32, i32, i32, P, P, P, i32, i32,
                                    i32, dbl, P, P]
        lib.orc_prefill.restype = ctypes.c_int
        lib.orc_e4m3_encode_array.argtypes = [P, i64, P]
        lib.orc_e4m3_encode_array.restype = None
        lib.orc_write_kv_cache_fp8.argtypes = [P, P, P, P, P, i32, f32, f32, i32, i32, i32, i32]
        lib.orc_write_kv_cache_fp8.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return 0
    if a.dtype == np.uint16:
        return 1
    if a.dtype == np.uint8:
        return 2  # E4M3 codes
    if a.dtype == np.float64:
        return 3
    raise TypeError("storage dtype must be float32, uint16 (bf16 bits), uint8 (E4M3 codes) "
                    f"or float64, got {a.dtype}")


def set_num_threads(n: int) -> None:
    """Threads of the oracle's OpenMP loops from now on (timing runs)."""
    _load().orc_set_num_threads(int(n))


def max_threads() -> int:
    """Threads the oracle's OpenMP loops use."""
    return int(_load().orc_max_threads())


def e4m3_value(codes: np.ndarray) -> np.ndarray:
    """E4M3 codes (uint8) -> their exact values as float64 (OCP 8-bit
    floating point E4M3, "fn" form: bias 7, subnormals at exponent 0, no
    infinities, S.1111.111 is NaN; largest finite 448)."""
    return widen(np.ascontiguousarray(codes, dtype=np.uint8))


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """The E4M3 code nearest to each value (ties to the even mantissa,
    magnitudes >= 448 saturate to 448, NaN -> 0x7F)."""
    xs = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(xs.shape, dtype=np.uint8)
    _load().orc_e4m3_encode_array(_ptr(xs), xs.size, _ptr(out))
    return out


def dequantize(codes: np.ndarray, scale: float) -> np.ndarray:
    """FP8 pages as the values they stand for: code value * scale, in
    float64 (exact: a code has at most 4 significant bits, a float32 scale
    24)."""
    return e4m3_value(codes) * np.float64(np.float32(scale))


def write_kv_cache_fp8(key_cache: np.ndarray, value_cache: np.ndarray, k_new: np.ndarray,
                       v_new: np.ndarray, slot_mapping: np.ndarray, k_scale: float,
                       v_scale: float) -> int:
    """Cache write into FP8 pages, in place: each element of the bf16 rows
    k_new / v_new [N, Hkv, D] (uint16 bits) is divided by its scale in IEEE
    single precision and rounded to the nearest E4M3 code, then stored at
    its slot as in write_kv_cache (teaching page, "Writing slots and reading
    the block table must agree").  Returns flags."""
    NB, bs, Hkv, D = key_cache.shape
    assert key_cache.dtype == np.uint8 and value_cache.dtype == np.uint8
    assert k_new.dtype == np.uint16 and v_new.dtype == np.uint16
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    kn = np.ascontiguousarray(k_new)
    vn = np.ascontiguousarray(v_new)
    return _load().orc_write_kv_cache_fp8(_ptr(key_cache), _ptr(value_cache), _ptr(kn), _ptr(vn),
                                          _ptr(sm), sm.size, np.float32(k_scale),
                                          np.float32(v_scale), NB, bs, Hkv, D)


def decode_fp8(q, key_cache, value_cache, k_scale: float, v_scale: float, block_tables,
               context_lens, scale: Optional[float] = None):
    """decode() over FP8 pages: the pages stand for code * scale (per
    tensor) and q is bf16 (uint16 bits); every value is widened exactly to
    float64 first.  Returns (out [B, Hq, D] float64, flags [B])."""
    assert key_cache.dtype == np.uint8 and q.dtype == np.uint16
    return decode(widen(q), dequantize(key_cache, k_scale), dequantize(value_cache, v_scale),
                  block_tables, context_lens, scale)


def map_token(block_table, token_index: int, block_size: int, num_blocks: int
              ) -> Tuple[int, int, int]:
    """Logical token -> (physical_block_id, block_offset, flags).

    Page "Implementing teaching PagedAttention: reading the historical KV
    cache from the block table", section "From logical token to physical
    block": logical_block_id = t // block_size, block_offset =
    t % block_size, physical_block_id = block_table[logical_block_id]."""
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    pb = ctypes.c_int32(-1)
    off = ctypes.c_int32(-1)
    f = _load().orc_map_token(_ptr(bt), bt.size, num_blocks, block_size, token_index,
                              ctypes.byref(pb), ctypes.byref(off))
    return pb.value, off.value, f


def widen(stored: np.ndarray) -> np.ndarray:
    """Stored float32 / bf16-bit values widened exactly to float64."""
    s = np.ascontiguousarray(stored)
    out = np.empty(s.shape, dtype=np.float64)
    _load().orc_widen(_ptr(s), _dtype_code(s), s.size, _ptr(out))
    return out


def gather_kv(key_cache, value_cache, block_table, context_len: int):
    """Paged gather of one sequence's K/V into logical order, as float64
    [context_len, Hkv, D] (teaching page, "Paged gather for a single
    Sequence").  Returns (keys, values, flags)."""
    NB, bs, Hkv, D = key_cache.shape
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    keys = np.zeros((max(context_len, 0), Hkv, D), dtype=np.float64)
    vals = np.zeros_like(keys)
    f = _load().orc_gather_kv(_ptr(key_cache), _ptr(value_cache), _dtype_code(key_cache),
                              NB, bs, Hkv, D, _ptr(bt), bt.size, context_len,
                              _ptr(keys), _ptr(vals))
    return keys, vals, f


def attention(q: np.ndarray, keys: np.ndarray, values: np.ndarray, scale: float) -> np.ndarray:
    """Standard softmax attention of one decode query on contiguous K/V:
    q [Hq, D] float64, keys/values [ctx, Hkv, D] float64 -> [Hq, D].

    Optimisation-route page, "What the attention kernel really does":
    score_i = dot(query, key_i) * scale, softmax, weighted sum of values."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    keys = np.ascontiguousarray(keys, dtype=np.float64)
    values = np.ascontiguousarray(values, dtype=np.float64)
    Hq, D = q.shape
    ctx, Hkv, D2 = keys.shape
    assert D == D2 and Hq % Hkv == 0
    out = np.empty((Hq, D), dtype=np.float64)
    _load().orc_attention(_ptr(q), _ptr(keys), _ptr(values), ctx, Hq, Hkv, D, scale, _ptr(out))
    return out


def decode(q, key_cache, value_cache, block_tables, context_lens, scale: Optional[float] = None):
    """Batched paged decode: gather then standard attention per sequence.
    Returns (out [B, Hq, D] float64, per-sequence flags [B] int32).

    Teaching page, "Extending to a batch: every Sequence has its own block
    table"; zero output for flagged or empty sequences."""
    B, Hq, D = q.shape
    NB, bs, Hkv, _ = key_cache.shape
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    if scale is None:
        scale = 1.0 / float(np.sqrt(D))
    out = np.empty((B, Hq, D), dtype=np.float64)
    flags = np.zeros(B, dtype=np.int32)
    _load().orc_decode(_ptr(q), _ptr(key_cache), _ptr(value_cache), _dtype_code(key_cache),
                       NB, bs, Hkv, D, _ptr(bt), _ptr(cl), B, Hq, bt.shape[1], scale,
                       _ptr(out), _ptr(flags))
    return out, flags


def partials(q, key_cache, value_cache, block_tables, context_lens, partition_tokens: int,
             max_partitions: int, scale: Optional[float] = None):
    """Per-partition (max, sum, normalised partial output) in float64:
    part_max/part_sum [B, Hq, P], part_out [B, Hq, P, D].  Empty partitions
    carry (-inf, 0, 0).  Returns (part_max, part_sum, part_out, flags)."""
    B, Hq, D = q.shape
    NB, bs, Hkv, _ = key_cache.shape
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    if scale is None:
        scale = 1.0 / float(np.sqrt(D))
    pm = np.empty((B, Hq, max_partitions), dtype=np.float64)
    ps = np.empty_like(pm)
    po = np.empty((B, Hq, max_partitions, D), dtype=np.float64)
    f = _load().orc_partials(_ptr(q), _ptr(key_cache), _ptr(value_cache),
                             _dtype_code(key_cache), NB, bs, Hkv, D, _ptr(bt), _ptr(cl), B, Hq,
                             bt.shape[1], scale, partition_tokens, max_partitions,
                             _ptr(pm), _ptr(ps), _ptr(po))
    return pm, ps, po, f


def merge(part_max, part_sum, part_out) -> np.ndarray:
    """Merge partials: M = max m_p, w_p = l_p exp(m_p - M),
    out = sum w_p o_p / sum w_p (zeros when no partition is non-empty)."""
    pm = np.ascontiguousarray(part_max, dtype=np.float64)
    ps = np.ascontiguousarray(part_sum, dtype=np.float64)
    po = np.ascontiguousarray(part_out, dtype=np.float64)
    B, Hq, P, D = po.shape
    out = np.empty((B, Hq, D), dtype=np.float64)
    _load().orc_merge(_ptr(pm), _ptr(ps), _ptr(po), B, Hq, D, P, _ptr(out))
    return out


def write_kv_cache(key_cache, value_cache, k_new, v_new, slot_mapping) -> int:
    """Byte copy of each new token's K/V row to its slot (in place).
    Teaching page, "Writing slots and reading the block table must agree".
    Returns flags (FLAG_SLOT for a slot past the pool)."""
    NB, bs, Hkv, D = key_cache.shape
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    kn = np.ascontiguousarray(k_new, dtype=key_cache.dtype)
    vn = np.ascontiguousarray(v_new, dtype=key_cache.dtype)
    return _load().orc_write_kv_cache(_ptr(key_cache), _ptr(value_cache), _ptr(kn), _ptr(vn),
                                      _ptr(sm), sm.size, key_cache.itemsize, NB, bs, Hkv, D)


def prefill(q, key_cache, value_cache, block_tables, context_lens, query_start,
            scale: Optional[float] = None):
    """Paged (chunked) prefill with the causal mask (teaching page, "Where is
    the attention mask"; route page, "decode attention and prefill attention
    are different").  Sequence b's new tokens are rows query_start[b] ..
    query_start[b+1]-1 of q [T, Hq, D]; their K/V are already stored at their
    slots, its history holds context_lens[b] tokens including them, and new
    token j (position context_lens[b] - n_b + j) attends to positions 0..that
    position through the block table.  Returns (out [T, Hq, D] float64,
    flags [B])."""
    NB, bs, Hkv, D = key_cache.shape
    T, Hq, Dq = q.shape
    assert Dq == D and q.dtype == key_cache.dtype
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    qs = np.ascontiguousarray(query_start, dtype=np.int32)
    B = cl.size
    assert qs.size == B + 1 and qs[-1] == T
    qq = np.ascontiguousarray(q)
    out = np.zeros((T, Hq, D), dtype=np.float64)
    flags = np.zeros(B, dtype=np.int32)
    _load().orc_prefill(_ptr(qq), _ptr(key_cache), _ptr(value_cache), _dtype_code(key_cache),
                        NB, bs, Hkv, D, _ptr(bt), _ptr(cl), _ptr(qs), B, Hq, bt.shape[1],
                        float(scale), _ptr(out), _ptr(flags))
    return out, flags

