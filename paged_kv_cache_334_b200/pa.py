"""Thin ctypes binding of libpa (the C ABI declared in include/pa.h).

Argument marshalling only: torch tensors are used for device memory and
streams, their pointers and sizes are handed to the library, and a non-OK
status raises :class:`PaError`.  Every step of the computation runs in the
CUDA kernels of ``libpa.so``; there is no CPU fallback, and importing the
library fails loudly when it has not been built.

The function names match the C entry points.  Shapes (row-major, dense):

* ``key_cache``, ``value_cache``: ``[num_blocks, block_size, num_kv_heads, head_dim]``
* ``q``, ``out``: ``[batch, num_q_heads, head_dim]``
* ``k_new``, ``v_new``: ``[num_tokens, num_kv_heads, head_dim]``
* ``block_tables``: ``[batch, max_blocks_per_seq]`` int32
* ``context_lens``: ``[batch]`` int32; ``slot_mapping``: ``[num_tokens]`` int64
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")

PA_OK = 0
PA_ERR_INVALID_ARG = 1
PA_ERR_UNSUPPORTED = 2
PA_ERR_CUDA = 3
PA_DTYPE_F32 = 0
PA_DTYPE_BF16 = 1
PA_DTYPE_FP8_E4M3 = 2  # E4M3 codes; q, out and new rows bf16
PA_DEVERR_BLOCK_ID = 1
PA_DEVERR_CONTEXT_LEN = 2
PA_DEVERR_SLOT = 4
PA_DEVERR_TIMEOUT = 8
PA_DEVERR_PREFIX = 16

EXPORTED_SYMBOLS = (
    "pa_version", "pa_status_string", "pa_last_error_message", "pa_write_kv_cache",
    "pa_decode_workspace_bytes", "pa_decode", "pa_decode_splitk", "pa_reduce",
    "pa_decode_noalloc", "pa_forward_decode", "pa_decode_shared_prefix",
    "pa_decode_shared_prefix_workspace_bytes", "pa_prefill",
)

# Size of the fixed device scratch array pa_decode_noalloc uses.
NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024


class PaError(RuntimeError):
    """A libpa call returned a non-OK status."""

    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


class CacheDesc(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("k_scale", ctypes.c_float),
                ("v_scale", ctypes.c_float)]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libpa.so and declare the entry points' signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m paged_kv_cache_334_b200.build` (there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    P, i32, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    D = ctypes.POINTER(CacheDesc)
    lib.pa_version.argtypes = []
    lib.pa_version.restype = i32
    lib.pa_status_string.argtypes = [i32]
    lib.pa_status_string.restype = ctypes.c_char_p
    lib.pa_last_error_message.argtypes = []
    lib.pa_last_error_message.restype = ctypes.c_char_p
    lib.pa_write_kv_cache.argtypes = [D, P, P, P, P, P, i32, P, P]
    lib.pa_write_kv_cache.restype = ctypes.c_int
    lib.pa_decode_workspace_bytes.argtypes = [D, i32, i32, i32]
    lib.pa_decode_workspace_bytes.restype = sz
    lib.pa_decode.argtypes = [D, P, P, P, P, P, P, i32, i32, i32, f32, P, sz, P, P]
    lib.pa_decode.restype = ctypes.c_int
    lib.pa_decode_splitk.argtypes = [D, P, P, P, P, P, i32, i32, i32, f32, i32, i32, P, P, P, P, P]
    lib.pa_decode_splitk.restype = ctypes.c_int
    lib.pa_reduce.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32, P, P]
    lib.pa_reduce.restype = ctypes.c_int
    lib.pa_decode_noalloc.argtypes = [D, P, P, P, P, P, P, i32, i32, i32, f32, P, P]
    lib.pa_decode_noalloc.restype = ctypes.c_int
    lib.pa_forward_decode.argtypes = [D, P, P, P, P, P, P, P, P, P, i32, i32, i32, f32, P, sz,
                                      P, P]
    lib.pa_forward_decode.restype = ctypes.c_int
    lib.pa_decode_shared_prefix_workspace_bytes.argtypes = [D, i32, i32, i32, i32]
    lib.pa_decode_shared_prefix_workspace_bytes.restype = sz
    lib.pa_decode_shared_prefix.argtypes = [D, P, P, P, P, P, P, i32, i32, i32, i32, f32, P, sz,
                                            P, P]
    lib.pa_decode_shared_prefix.restype = ctypes.c_int
    lib.pa_prefill.argtypes = [D, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, f32, P, P]
    lib.pa_prefill.restype = ctypes.c_int
    _lib = lib
    return lib


def _check(status: int) -> None:
    if status != PA_OK:
        lib = load()
        raise PaError(status, f"{lib.pa_status_string(status).decode()}: "
                              f"{lib.pa_last_error_message().decode()}")


def _dtype_code(dtype: torch.dtype) -> int:
    if dtype == torch.float32:
        return PA_DTYPE_F32
    if dtype == torch.bfloat16:
        return PA_DTYPE_BF16
    if dtype == torch.float8_e4m3fn:
        return PA_DTYPE_FP8_E4M3
    raise TypeError(f"unsupported dtype {dtype}: libpa takes float32, bfloat16 or "
                    "float8_e4m3fn (caches)")


def _dev(t: Optional[torch.Tensor], name: str, dtype: Optional[torch.dtype] = None):
    """Pointer of a dense CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise TypeError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr()) if t.numel() else None


def _act(key_cache: torch.Tensor) -> torch.dtype:
    """dtype of q, out and the new rows for this cache (bf16 for FP8 pages)."""
    return torch.bfloat16 if key_cache.dtype == torch.float8_e4m3fn else key_cache.dtype


def cache_desc(key_cache: torch.Tensor, k_scale: float = 1.0, v_scale: float = 1.0) -> CacheDesc:
    """The pool's shape; k_scale / v_scale: FP8 pages stand for code * scale."""
    if key_cache.dim() != 4:
        raise ValueError("key_cache must be [num_blocks, block_size, num_kv_heads, head_dim]")
    nb, bs, hkv, d = key_cache.shape
    return CacheDesc(nb, bs, hkv, d, _dtype_code(key_cache.dtype), float(k_scale), float(v_scale))


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def pa_version() -> int:
    return int(load().pa_version())


def pa_write_kv_cache(key_cache, value_cache, k_new, v_new, slot_mapping,
                      err_word: Optional[torch.Tensor] = None, stream=None,
                      k_scale: float = 1.0, v_scale: float = 1.0) -> None:
    """Store each new token's K/V row at its slot (see include/pa.h)."""
    lib = load()
    desc = cache_desc(key_cache, k_scale, v_scale)
    if value_cache.shape != key_cache.shape or value_cache.dtype != key_cache.dtype:
        raise ValueError("value_cache must match key_cache")
    _check(lib.pa_write_kv_cache(
        ctypes.byref(desc), _dev(key_cache, "key_cache"), _dev(value_cache, "value_cache"),
        _dev(k_new, "k_new", _act(key_cache)), _dev(v_new, "v_new", _act(key_cache)),
        _dev(slot_mapping, "slot_mapping", torch.int64), int(slot_mapping.numel()),
        _dev(err_word, "err_word", torch.int32), _stream(stream)))


def pa_decode_workspace_bytes(key_cache, batch: int, num_q_heads: int,
                              max_blocks_per_seq: int,
                              k_scale: float = 1.0, v_scale: float = 1.0) -> int:
    desc = cache_desc(key_cache, k_scale, v_scale)
    return int(load().pa_decode_workspace_bytes(ctypes.byref(desc), batch, num_q_heads,
                                                max_blocks_per_seq))


_workspaces = {}


def decode_workspace(key_cache, batch: int, num_q_heads: int, max_blocks_per_seq: int,
                     k_scale: float = 1.0, v_scale: float = 1.0) -> torch.Tensor:
    """A zero-filled workspace for pa_decode, cached per device and size
    (pa_decode leaves it zero-filled, so it can be reused by stream-ordered
    calls)."""
    n = pa_decode_workspace_bytes(key_cache, batch, num_q_heads, max_blocks_per_seq,
                                  k_scale=k_scale, v_scale=v_scale)
    key = (key_cache.device, n)
    ws = _workspaces.get(key)
    if ws is None:
        ws = torch.zeros(max(n, 256), dtype=torch.uint8, device=key_cache.device)
        _workspaces[key] = ws
    return ws


def pa_decode(out, q, key_cache, value_cache, block_tables, context_lens,
              scale: Optional[float] = None, workspace: Optional[torch.Tensor] = None,
              err_word: Optional[torch.Tensor] = None, stream=None,
              k_scale: float = 1.0, v_scale: float = 1.0) -> torch.Tensor:
    """Fused paged decode attention into `out` (see include/pa.h)."""
    lib = load()
    desc = cache_desc(key_cache, k_scale, v_scale)
    B, Hq, Dq = q.shape
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    if scale is None:
        scale = 1.0 / math.sqrt(Dq)
    if workspace is None:
        workspace = decode_workspace(key_cache, B, Hq, MB, k_scale=k_scale, v_scale=v_scale)
    _check(lib.pa_decode(
        ctypes.byref(desc), _dev(out, "out", _act(key_cache)), _dev(q, "q", _act(key_cache)),
        _dev(key_cache, "key_cache"), _dev(value_cache, "value_cache", key_cache.dtype),
        _dev(block_tables, "block_tables", torch.int32),
        _dev(context_lens, "context_lens", torch.int32), B, Hq, MB, float(scale),
        _dev(workspace, "workspace"), int(workspace.numel() * workspace.element_size()),
        _dev(err_word, "err_word", torch.int32), _stream(stream)))
    return out


def pa_forward_decode(out, q, key_cache, value_cache, k_new, v_new, slot_mapping,
                      block_tables, context_lens, scale: Optional[float] = None,
                      workspace: Optional[torch.Tensor] = None,
                      err_word: Optional[torch.Tensor] = None, stream=None,
                      k_scale: float = 1.0, v_scale: float = 1.0) -> torch.Tensor:
    """One decode step: store each sequence's newest K/V row at its slot, then
    decode over the whole history into `out` (see include/pa.h)."""
    lib = load()
    desc = cache_desc(key_cache, k_scale, v_scale)
    B, Hq, Dq = q.shape
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    if slot_mapping.numel() != B:
        raise ValueError("slot_mapping must hold one slot per sequence")
    if scale is None:
        scale = 1.0 / math.sqrt(Dq)
    if workspace is None:
        workspace = decode_workspace(key_cache, B, Hq, MB, k_scale=k_scale, v_scale=v_scale)
    _check(lib.pa_forward_decode(
        ctypes.byref(desc), _dev(out, "out", _act(key_cache)), _dev(q, "q", _act(key_cache)),
        _dev(key_cache, "key_cache"), _dev(value_cache, "value_cache", key_cache.dtype),
        _dev(k_new, "k_new", _act(key_cache)), _dev(v_new, "v_new", _act(key_cache)),
        _dev(slot_mapping, "slot_mapping", torch.int64),
        _dev(block_tables, "block_tables", torch.int32),
        _dev(context_lens, "context_lens", torch.int32), B, Hq, MB, float(scale),
        _dev(workspace, "workspace"), int(workspace.numel() * workspace.element_size()),
        _dev(err_word, "err_word", torch.int32), _stream(stream)))
    return out


def pa_decode_shared_prefix(out, q, key_cache, value_cache, block_tables, context_lens,
                            prefix_blocks: int, scale: Optional[float] = None,
                            workspace: Optional[torch.Tensor] = None,
                            err_word: Optional[torch.Tensor] = None, stream=None,
                            k_scale: float = 1.0, v_scale: float = 1.0) -> torch.Tensor:
    """pa_decode for a batch whose tables all start with the same
    prefix_blocks pages (see include/pa.h)."""
    lib = load()
    desc = cache_desc(key_cache, k_scale, v_scale)
    B, Hq, Dq = q.shape
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    if scale is None:
        scale = 1.0 / math.sqrt(Dq)
    if workspace is None:
        n = int(lib.pa_decode_shared_prefix_workspace_bytes(ctypes.byref(desc), B, Hq, MB,
                                                            int(prefix_blocks)))
        key = (key_cache.device, n, "prefix")
        workspace = _workspaces.get(key)
        if workspace is None:
            workspace = torch.zeros(max(n, 256), dtype=torch.uint8, device=key_cache.device)
            _workspaces[key] = workspace
    _check(lib.pa_decode_shared_prefix(
        ctypes.byref(desc), _dev(out, "out", _act(key_cache)), _dev(q, "q", _act(key_cache)),
        _dev(key_cache, "key_cache"), _dev(value_cache, "value_cache", key_cache.dtype),
        _dev(block_tables, "block_tables", torch.int32),
        _dev(context_lens, "context_lens", torch.int32), B, Hq, MB, int(prefix_blocks),
        float(scale), _dev(workspace, "workspace"),
        int(workspace.numel() * workspace.element_size()), _dev(err_word, "err_word", torch.int32),
        _stream(stream)))
    return out


def pa_decode_splitk(q, key_cache, value_cache, block_tables, context_lens,
                     partition_tokens: int, part_max, part_sum, part_out,
                     scale: Optional[float] = None, err_word: Optional[torch.Tensor] = None,
                     stream=None,
                     k_scale: float = 1.0, v_scale: float = 1.0) -> None:
    """Per-partition (max, sum, normalised output) partials (see include/pa.h).
    part_max/part_sum: [B, Hq, P] float32; part_out: [B, Hq, P, D] float32."""
    lib = load()
    desc = cache_desc(key_cache, k_scale, v_scale)
    B, Hq, Dq = q.shape
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    P = part_max.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(Dq)
    _check(lib.pa_decode_splitk(
        ctypes.byref(desc), _dev(q, "q", _act(key_cache)), _dev(key_cache, "key_cache"),
        _dev(value_cache, "value_cache", key_cache.dtype),
        _dev(block_tables, "block_tables", torch.int32),
        _dev(context_lens, "context_lens", torch.int32), B, Hq, MB, float(scale),
        int(partition_tokens), int(P), _dev(part_max, "part_max", torch.float32),
        _dev(part_sum, "part_sum", torch.float32), _dev(part_out, "part_out", torch.float32),
        _dev(err_word, "err_word", torch.int32), _stream(stream)))


def pa_reduce(out, part_max, part_sum, part_out, context_lens, partition_tokens: int,
              err_word: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Merge partials into `out` [B, Hq, D] (see include/pa.h)."""
    lib = load()
    B, Hq, P, Dh = part_out.shape
    _check(lib.pa_reduce(
        _dev(out, "out"), _dev(part_max, "part_max", torch.float32),
        _dev(part_sum, "part_sum", torch.float32), _dev(part_out, "part_out", torch.float32),
        _dev(context_lens, "context_lens", torch.int32), B, Hq, Dh, int(partition_tokens),
        int(P), _dtype_code(out.dtype), _dev(err_word, "err_word", torch.int32),
        _stream(stream)))
    return out


def pa_decode_noalloc(out, q, key_cache, value_cache, block_tables, context_lens,
                      scale: Optional[float] = None, err_word: Optional[torch.Tensor] = None,
                      stream=None,
                      k_scale: float = 1.0, v_scale: float = 1.0) -> torch.Tensor:
    """pa_decode without a workspace, for callers that may not allocate device
    memory: the library's own fixed scratch array (NOALLOC_SCRATCH_BYTES per
    GPU) stands in for it.  Sizes whose workspace would not fit raise
    PaError(PA_ERR_UNSUPPORTED).  Calls that overlap on the GPU share that
    array and race; keep them on one stream (see include/pa.h)."""
    lib = load()
    desc = cache_desc(key_cache, k_scale, v_scale)
    B, Hq, Dq = q.shape
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    if scale is None:
        scale = 1.0 / math.sqrt(Dq)
    _check(lib.pa_decode_noalloc(
        ctypes.byref(desc), _dev(out, "out", _act(key_cache)), _dev(q, "q", _act(key_cache)),
        _dev(key_cache, "key_cache"), _dev(value_cache, "value_cache", key_cache.dtype),
        _dev(block_tables, "block_tables", torch.int32),
        _dev(context_lens, "context_lens", torch.int32), B, Hq, MB, float(scale),
        _dev(err_word, "err_word", torch.int32), _stream(stream)))
    return out


def pa_prefill(out, q, key_cache, value_cache, block_tables, context_lens, query_start,
               max_query_len: Optional[int] = None, scale: Optional[float] = None,
               err_word: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Paged (chunked) prefill with the causal mask into `out` [T, Hq, D]:
    sequence b's new tokens are rows query_start[b] .. query_start[b+1]-1 of
    q, their K/V already stored, context_lens[b] counting them (see
    include/pa.h).  max_query_len (>= every chunk's length) defaults to the
    longest chunk, which reads query_start back to the host."""
    lib = load()
    desc = cache_desc(key_cache)
    T, Hq, Dq = q.shape
    B = context_lens.numel()
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    if query_start.numel() != B + 1:
        raise ValueError("query_start must hold batch + 1 entries")
    if scale is None:
        scale = 1.0 / math.sqrt(Dq)
    if max_query_len is None:
        max_query_len = int((query_start[1:] - query_start[:-1]).max().item()) if B else 0
    _check(lib.pa_prefill(
        ctypes.byref(desc), _dev(out, "out", key_cache.dtype), _dev(q, "q", key_cache.dtype),
        _dev(key_cache, "key_cache"), _dev(value_cache, "value_cache", key_cache.dtype),
        _dev(block_tables, "block_tables", torch.int32),
        _dev(context_lens, "context_lens", torch.int32),
        _dev(query_start, "query_start", torch.int32), B, T, Hq, MB, int(max_query_len),
        float(scale), _dev(err_word, "err_word", torch.int32), _stream(stream)))
    return out
