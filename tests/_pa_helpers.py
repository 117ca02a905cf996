"""Shared helpers for the GPU tests: move a seeded workload to the device, run
the hot path through the C ABI, and compare against the fp64 oracle."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from paged_kv_cache_334_b200 import pa
from paged_kv_cache_334_b200 import workloads as wl

# Tolerances against the fp64 oracle.
F32_MAX_ABS = 1e-5
BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 1e-2


def torch_dtype(w):
    return torch.float32 if w.dtype == wl.DTYPE_F32 else torch.bfloat16


def to_dev(arr: np.ndarray, dtype: str, device="cuda"):
    t = torch.from_numpy(np.ascontiguousarray(arr))
    if arr.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t.to(device)


def upload(w, device="cuda"):
    d = {
        "q": to_dev(w.q, w.dtype, device),
        "key_cache": to_dev(w.key_cache, w.dtype, device),
        "value_cache": to_dev(w.value_cache, w.dtype, device),
        "block_tables": torch.from_numpy(w.block_tables).to(device),
        "context_lens": torch.from_numpy(w.context_lens).to(device),
    }
    if w.slot_mapping is not None:
        d["k_new"] = to_dev(w.k_new, w.dtype, device)
        d["v_new"] = to_dev(w.v_new, w.dtype, device)
        d["slot_mapping"] = torch.from_numpy(w.slot_mapping).to(device)
    return d


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def oracle_after_write(w):
    """The oracle's own write of the new tokens followed by its decode."""
    kc, vc = w.key_cache.copy(), w.value_cache.copy()
    if w.slot_mapping is not None:
        assert oracle.write_kv_cache(kc, vc, w.k_new, w.v_new, w.slot_mapping) == 0
    out, flags = oracle.decode(w.q, kc, vc, w.block_tables, w.context_lens,
                               1.0 / math.sqrt(w.head_dim))
    return out, flags, kc, vc


def gpu_write_and_decode(w, d, err=None):
    if "slot_mapping" in d:
        pa.pa_write_kv_cache(d["key_cache"], d["value_cache"], d["k_new"], d["v_new"],
                             d["slot_mapping"], err_word=err)
    out = torch.empty_like(d["q"])
    pa.pa_decode(out, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                 d["context_lens"], err_word=err)
    return out


def assert_close(got: np.ndarray, ref: np.ndarray, dtype: str, what=""):
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    if dtype == wl.DTYPE_F32:
        assert err.max() <= F32_MAX_ABS, f"{what}: max abs err {err.max():.3e} > {F32_MAX_ABS}"
    else:
        assert err.max() <= BF16_MAX_ABS, f"{what}: max abs err {err.max():.3e} > {BF16_MAX_ABS}"
        assert err.mean() <= BF16_MEAN_ABS, f"{what}: mean abs err {err.mean():.3e}"
    return float(err.max()), float(err.mean())
