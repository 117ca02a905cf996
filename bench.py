#!/usr/bin/env python
"""Benchmark of one paged decode-attention step on B200.

A step is one pass of the hot path over one batch: the cache write of every
sequence's newest token via slot_mapping followed by the fused paged decode,
through the C ABI -- by default as one pa_forward_decode call (the write
happens inside the decode kernel), with ``--step separate`` as
pa_write_kv_cache followed by pa_decode.  The default workload is
mixed_bf16 (128 sequences of 128 / 4096 / 16000 tokens, 32 query / 8 KV
heads, head_dim 128, block_size 16, 2.58 GB of pages), and the same line
carries a second record (``--companion``, default gqa_bf16: batch 32,
context lengths uniform in [128, 2048]); other workloads are selectable with
--workload.  ``--step splitk`` times pa_write_kv_cache, pa_decode_splitk and
pa_reduce (long_bf16 by default), ``--step prefix`` pa_write_kv_cache and
pa_decode_shared_prefix (mqa_prefix_bf16 by default).

Output: one JSON line on rank 0.  ``value`` is the achieved bandwidth on the
algorithmic bytes of the step (unique K/V bytes of the visible tokens, block
tables, context lengths, q, out and the new K/V rows) in GB/s, summed over
ranks and divided by the slowest rank's time; each timed step is preceded by
an L2 flush outside its CUDA-event pair, and a 20 ms device sleep before the
first timed step keeps the host's launches ahead of the device.  ``e2e`` is the same metric with the
per-step inputs copied from pinned host memory and the output read back
inside the timed region.  ``roofline`` reports the decode call (the whole
step when fused) against the measured HBM copy bandwidth; ``cpu_baseline`` times the fp64 CPU
oracle on the host cores (rank 0, one GPU only).

Multi-GPU (torchrun, one process per GPU): every rank decodes its own
independent batch (seeded by rank); there is no data-path collective, only a
barrier and max/sum reductions of the timings (weak scaling).

``--impl reference`` times the fp64 CPU oracle itself as the reference arm
(rank 0 only; other ranks exit at once).

``--step prefill`` measures pa_prefill instead: the workload's sequences as
whole prompts (or, with ``--chunk C``, the last C tokens of each context as
a later chunk), all their K/V in the pool, one call per step, reported in
TFLOP/s of causal attention (QK and PV of every visible position) against
the measured bf16 tensor peak.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from paged_kv_cache_334_b200 import workloads as wl  # noqa: E402

METRIC = "decode-attention KV GB/s & fraction of B200 HBM peak; seq-tokens/s per step"
FALLBACK_HBM_GBS = 6650.0
CSRC = os.path.join(ROOT, "paged_kv_cache_334_b200", "csrc")
# sources that define the decode kernel's code and launch shape
DECODE_SOURCES = ("decode_stream.cuh", "decode_stream_bf16.cu", "decode_stream_f32.cu",
                  "decode_stream_fp8.cu", "reduce.cu", "sm100_ptx.cuh", "pa_common.cuh",
                  "pa_launch.h", "api.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.md")


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=None, choices=wl.WORKLOADS,
                    help="default: the mixed-length continuous batch (decode steps), the "
                         "long-context batch (--step splitk), the bf16 GQA batch as prompts "
                         "(--step prefill)")
    ap.add_argument("--companion", default="gqa_bf16", choices=wl.WORKLOADS + ("none",),
                    help="a second workload measured in the same run and reported under its "
                         "own key of the same JSON line (default: the bf16 GQA batch, the "
                         "other configuration the target names); 'none' skips it")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--batch", type=int, default=None,
                    help="the workload's first BATCH sequences only (smaller captures for "
                         "profiling; not a headline configuration)")
    ap.add_argument("--block-size", type=int, default=None,
                    help="page size override for gqa_bf16 / mixed_bf16 / long_bf16 (a sweep)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--step", choices=("fused", "separate", "prefix", "splitk", "prefill"),
                    default="fused",
                    help="fused: one pa_forward_decode call per step (cache write inside the "
                         "decode kernel); separate: pa_write_kv_cache then pa_decode; prefix: "
                         "pa_write_kv_cache then pa_decode_shared_prefix (workloads with a "
                         "shared prefix); splitk: pa_write_kv_cache then pa_decode_splitk "
                         "(--partition-tokens partitions) and pa_reduce; prefill: one "
                         "pa_prefill call over the workload's sequences as whole prompts "
                         "(bf16 workloads), reported in TFLOP/s")
    ap.add_argument("--partition-tokens", type=int, default=512,
                    help="--step splitk: tokens per partition")
    ap.add_argument("--chunk", type=int, default=None,
                    help="--step prefill: the last CHUNK tokens of each context are the "
                         "chunk (a later chunk of a chunked prefill) instead of whole prompts")
    args = ap.parse_args(argv)
    if args.workload is None:
        args.workload = {"prefill": "gqa_bf16", "splitk": "long_bf16",
                         "prefix": "mqa_prefix_bf16"}.get(args.step, "mixed_bf16")
    return args


# ---------------------------------------------------------------------------
# ranks
# ---------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_seed(seed: int, rank: int) -> int:
    """Each rank decodes its own independent batch."""
    return seed + 1000 * rank


def init_dist(world: int, local: int, backend: str = "nccl"):
    import torch
    import torch.distributed as dist
    if world <= 1:
        return None
    kw = {}
    if backend == "nccl":
        kw["device_id"] = torch.device("cuda", local)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return dist


def reduce_scalar(x: float, op: str, dist=None, device=None) -> float:
    """max / sum of a host scalar over ranks (identity with one rank)."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.sel = str(device_index)

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.sel, "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "20", "-f", self.path],
                stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            deadline = time.time() + 3.0
            while time.time() < deadline and os.path.getsize(self.path) == 0:
                time.sleep(0.01)
        except Exception:
            self.proc = None

    def mark(self, which: str):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.05)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    rows.append((ts, float(parts[1]), float(parts[2]), parts[3], parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        inside = [r for r in rows if self.t0 is not None and self.t0 - 0.02 <= r[0] <= self.t1 + 0.02]
        note = "samples inside the timed region"
        if not inside:
            after = [r for r in rows if self.t0 is not None and r[0] >= self.t0]
            inside = after[:1] or rows[-1:]
            note = "timed region shorter than the 20 ms sampling period: nearest sample"
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in inside for n, v in zip(names, r[4]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside), "reasons": reasons,
                "samples": len(inside), "note": note}


# ---------------------------------------------------------------------------
# measured peaks and ncu traffic
# ---------------------------------------------------------------------------

def tensor_path(w) -> bool:
    """The shapes libpa decodes on tcgen05 tiles (64 or 128 query heads per
    KV head, bf16, head_dim 64 or 128, block_size 8..128)."""
    return (w.dtype == wl.DTYPE_BF16 and w.group in (64, 128) and w.head_dim in (64, 128)
            and 8 <= w.block_size <= 128)


def tensor_peak():
    """Dense bf16 tensor-core peak (burst: the call is timed alone)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "MEASURED_PEAKS.json bf16_tflops (of measured)"
    except Exception:
        return 1590.0, "1.59 PFLOP/s fallback (of fallback)"


def attention_flops(w) -> float:
    """QK and PV of every visible (token, query head): 2 * 2 * D flops each."""
    return 4.0 * float(w.context_lens.sum()) * w.num_q_heads * w.head_dim


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "MEASURED_PEAKS.json hbm_gbs (of measured)"
    except Exception:
        return FALLBACK_HBM_GBS, "6.65 TB/s fallback (of fallback)"


def _code_only(text: str) -> str:
    """C/C++ source without comments and blank-line or indentation
    differences, so that editing a comment keeps the recorded counters."""
    out, i, n = [], 0, len(text)
    while i < n:
        if text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif text[i] in "\"'":
            q, j = text[i], i + 1
            while j < n and text[j] != q:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            out.append(text[i])
            i += 1
    lines = (ln.strip() for ln in "".join(out).splitlines())
    return "\n".join(ln for ln in lines if ln)


def decode_source_hash() -> str:
    """Hash of the decode kernel's code (kernel, device helpers, launch plan),
    comments excluded."""
    h = hashlib.sha256()
    for name in DECODE_SOURCES:
        with open(os.path.join(CSRC, name), encoding="utf-8") as f:
            h.update(name.encode() + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


RUNWAY_NOTE = ("CUDA events around every step on the launching stream; a 20 ms device "
               "sleep before the first step keeps the host's launches ahead of the device")


def host_runway(ms: float = 20.0):
    """Keep the device busy for about `ms` before a timed loop, so that the
    host enqueues the first steps ahead of the device and no step's events
    wait on the host's launches: the events then bracket device work only
    (nothing is skipped; the runway sits outside every event pair)."""
    import torch
    torch.cuda._sleep(int(ms * 1e-3 * 2.0e9))


def staged_inputs(tensors, dev):
    """One device buffer and one pinned host buffer holding copies of
    `tensors` back to back (each 256-byte aligned), as a serving loop stages
    a step's inputs: a step's host-to-device transfer is then one copy.
    Returns (device buffer, host buffer, device views shaped like the
    tensors; the library is called on the views)."""
    import torch
    offs, pos = [], 0
    for t in tensors:
        offs.append(pos)
        pos += (t.numel() * t.element_size() + 255) // 256 * 256
    dev_buf = torch.zeros(max(pos, 256), dtype=torch.uint8, device=dev)
    host_buf = torch.zeros(max(pos, 256), dtype=torch.uint8).pin_memory()
    views = []
    for t, o in zip(tensors, offs):
        nb = t.numel() * t.element_size()
        raw = t.contiguous().view(torch.uint8).reshape(-1)
        host_buf[o:o + nb].copy_(raw.cpu())
        v = dev_buf[o:o + nb].view(t.dtype).view(t.shape)
        v.copy_(t)
        views.append(v)
    return dev_buf, host_buf, views


def recorded_traffic(workload: str):
    """DRAM bytes per decode call (all its kernels) from the committed ncu
    summary, if it was taken on the current kernel sources for this workload
    (`<workload>/splitk` for the split-K step); else None."""
    try:
        text = open(TRAFFIC_FILE).read()
    except OSError:
        return None
    want = decode_source_hash()
    for line in text.splitlines():
        parts = [p.strip() for p in line.strip().strip("|").split("|")]
        if len(parts) >= 3 and parts[0] == workload and parts[1] == want:
            try:
                return float(parts[2])
            except ValueError:
                return None
    return None


# ---------------------------------------------------------------------------
# the CPU oracle (baseline leg and reference arm)
# ---------------------------------------------------------------------------

def time_oracle(w, target_seconds: float, max_reps: int = 1000):
    """Time the fp64 oracle's step (its own cache write + decode) on the host
    cores, repeating the whole batch until about target_seconds elapsed, or
    on a prefix of the batch when one pass is longer than that."""
    import oracle
    oracle.build()
    sample = w
    t_one = _oracle_step(w)
    reps = 1
    desc = f"full {w.name} batch ({w.batch} sequences)"
    if t_one > target_seconds and w.batch > 1:
        nb = max(1, int(w.batch * target_seconds / t_one))
        sample = _prefix(w, nb)
        t_one = _oracle_step(sample)
        desc = f"first {nb} of {w.batch} sequences of {w.name}"
    total = t_one
    while total < target_seconds and reps < max_reps:
        total += _oracle_step(sample)
        reps += 1
    per_step = total / reps
    return per_step, sample, oracle.max_threads(), f"{desc}, {reps} repetition(s)"


def cpu_baseline(w, cpu_seconds: float) -> dict:
    """The oracle timed on the host cores (as many threads as its OpenMP
    loops get) on a bounded sample of the batch, and on one thread on the
    first 1/threads of that sample; GB/s on each sample's algorithmic
    bytes."""
    import oracle
    per_step, sample, threads, desc = time_oracle(w, cpu_seconds)
    line = {"value": wl.roofline_bytes(sample) / per_step / 1e9, "unit": "GB/s",
            "cores": threads, "kind": "oracle", "sample": desc,
            "ms_per_step": per_step * 1e3}
    nb1 = max(1, sample.batch // max(1, threads))
    one = _prefix(sample, nb1) if nb1 < sample.batch else sample
    oracle.set_num_threads(1)
    try:
        total, reps = _oracle_step(one), 1
        while total < cpu_seconds / 2 and reps < 1000:
            total += _oracle_step(one)
            reps += 1
    finally:
        oracle.set_num_threads(threads)
    line["single_thread"] = {
        "value": wl.roofline_bytes(one) / (total / reps) / 1e9, "unit": "GB/s", "cores": 1,
        "sample": f"first {nb1} of the {sample.batch} sequences above, {reps} repetition(s)",
        "ms_per_step": total / reps * 1e3}
    return line


SM_COUNT = 148
EX2_PER_SM_CLK = 16  # fp32 ex2 results per SM per clock (multi-function unit, nominal)


def ceilings(w, flops: float, nbytes: float, launch_us: float, sm_mhz: float) -> dict:
    """Lower bounds on one call's time from its three candidate limits --
    HBM bytes at the measured copy bandwidth, flops at the measured bf16
    peak, and one ex2 per (visible token, query head) score at the
    multi-function unit's nominal rate at the sampled SM clock -- and the
    call's time as a multiple of each."""
    hbm, _ = hbm_peak()
    tensor, _ = tensor_peak()
    exps = float(w.context_lens.sum()) * w.num_q_heads
    ex2_per_s = SM_COUNT * EX2_PER_SM_CLK * sm_mhz * 1e6
    out = {"hbm_us": nbytes / (hbm * 1e9) * 1e6,
           "tensor_us": flops / (tensor * 1e12) * 1e6,
           "ex2_us": exps / ex2_per_s * 1e6,
           "ex2_per_launch": exps, "ex2_peak_per_s": ex2_per_s,
           "ex2_peak": f"{SM_COUNT} SMs x {EX2_PER_SM_CLK} ex2/clock x {sm_mhz:.0f} MHz "
                       "(nominal unit count, sampled clock)",
           "launch_us": launch_us}
    for k in ("hbm", "tensor", "ex2"):
        out[k + "_frac"] = out[k + "_us"] / launch_us
    return out


def parity_sample(w, out_rows: np.ndarray, idx) -> dict:
    """Max / mean absolute difference between the timed call's output rows of
    the sequences `idx` (out_rows, float64, in that order) and the oracle's
    write then decode of those sequences, with the tolerance of the
    workload's dtype.  The write is idempotent, so the workload's host pool
    may already hold it."""
    import oracle
    s = _subset(w, idx)
    scale = 1.0 / math.sqrt(w.head_dim)
    kc, vc = s.key_cache, s.value_cache
    if w.dtype == wl.DTYPE_FP8:
        if s.slot_mapping is not None:
            oracle.write_kv_cache_fp8(kc, vc, s.k_new, s.v_new, s.slot_mapping, w.k_scale,
                                      w.v_scale)
        ref, flags = oracle.decode_fp8(s.q, kc, vc, w.k_scale, w.v_scale, s.block_tables,
                                       s.context_lens, scale)
    else:
        if s.slot_mapping is not None:
            oracle.write_kv_cache(kc, vc, s.k_new, s.v_new, s.slot_mapping)
        ref, flags = oracle.decode(s.q, kc, vc, s.block_tables, s.context_lens, scale)
    err = np.abs(np.asarray(out_rows, dtype=np.float64) - ref)
    tol_max, tol_mean = (1e-5, None) if w.dtype == wl.DTYPE_F32 else (2e-2, 1e-2)
    finite = bool(np.isfinite(err).all())
    ok = finite and not flags.any() and err.max() <= tol_max and (
        tol_mean is None or err.mean() <= tol_mean)
    return {"max_abs": float(err.max()), "mean_abs": float(err.mean()),
            "sequences": [int(i) for i in idx],
            "tolerance": {"max_abs": tol_max, "mean_abs": tol_mean}, "within": bool(ok)}


def parity_indices(batch: int, n: int = 12):
    """n sequences spread over the batch (its first and last included), so
    that sequences cut between CTAs and sequences kept whole are both
    checked."""
    return sorted(set(int(round(x)) for x in np.linspace(0, batch - 1, min(n, batch))))


def timing_stats(ms) -> dict:
    """Mean, median, minimum and maximum of per-step times (ms)."""
    ms = list(ms)
    return {"mean": statistics.mean(ms), "median": statistics.median(ms), "min": min(ms),
            "max": max(ms)}


def _oracle_step(w) -> float:
    import oracle
    kc, vc = w.key_cache, w.value_cache
    scale = 1.0 / math.sqrt(w.head_dim)
    t0 = time.perf_counter()
    if w.dtype == wl.DTYPE_FP8:
        if w.slot_mapping is not None:
            oracle.write_kv_cache_fp8(kc, vc, w.k_new, w.v_new, w.slot_mapping, w.k_scale,
                                      w.v_scale)
        oracle.decode_fp8(w.q, kc, vc, w.k_scale, w.v_scale, w.block_tables, w.context_lens,
                          scale)
        return time.perf_counter() - t0
    if w.slot_mapping is not None:
        oracle.write_kv_cache(kc, vc, w.k_new, w.v_new, w.slot_mapping)
    oracle.decode(w.q, kc, vc, w.block_tables, w.context_lens, scale)
    return time.perf_counter() - t0


def _subset(w, idx):
    """The workload restricted to sequences idx (same pool)."""
    import dataclasses
    idx = np.asarray(idx, dtype=np.int64)
    keep = w.slot_mapping is not None
    # the bench workloads have a new token in every sequence: row b is b's
    assert not keep or w.slot_mapping.shape[0] == w.batch
    return dataclasses.replace(
        w, batch=len(idx), q=w.q[idx].copy(), block_tables=w.block_tables[idx].copy(),
        context_lens=w.context_lens[idx].copy(),
        k_new=w.k_new[idx].copy() if keep else None, v_new=w.v_new[idx].copy() if keep else None,
        slot_mapping=w.slot_mapping[idx].copy() if keep else None)


def _prefix(w, nb):
    import dataclasses
    keep = w.slot_mapping is not None
    return dataclasses.replace(
        w, batch=nb, q=w.q[:nb].copy(), block_tables=w.block_tables[:nb].copy(),
        context_lens=w.context_lens[:nb].copy(),
        k_new=w.k_new[:nb].copy() if keep else None, v_new=w.v_new[:nb].copy() if keep else None,
        slot_mapping=w.slot_mapping[:nb].copy() if keep else None)


def workload_config(w, args):
    return {
        "workload": f"{w.name}: {w.description}",
        "batch": w.batch, "num_q_heads": w.num_q_heads, "num_kv_heads": w.num_kv_heads,
        "head_dim": w.head_dim, "block_size": w.block_size, "num_blocks": w.num_blocks,
        "context_tokens": int(w.context_lens.sum()), "seed": args.seed,
        "step": {"fused": "pa_forward_decode (newest token of every sequence stored inside the "
                          "decode kernel, then decode)",
                 "separate": "pa_write_kv_cache(newest token of every sequence) + pa_decode",
                 "prefix": "pa_write_kv_cache(newest token of every sequence) + "
                           "pa_decode_shared_prefix",
                 "splitk": f"pa_write_kv_cache(newest token of every sequence) + "
                           f"pa_decode_splitk({args.partition_tokens}-token partitions) + "
                           f"pa_reduce"}[args.step],
        "l2": "flushed before every timed step (zero-fill then read of 2x L2, outside the events)",
        "parallelism": f"replicas: one independent batch per GPU x{args.gpus}",
    }


def run_reference(args):
    world, rank, local = dist_env()
    if rank != 0:
        return 0
    w = wl.make_workload(args.workload, seed=args.seed, batch=args.batch,
                         block_size=args.block_size)
    nbytes_full = wl.roofline_bytes(w)
    budget = max(2.0, min(args.cpu_seconds, 150.0 / max(1, args.steps + args.warmup)))
    per_step, sample, cores, desc = time_oracle(w, budget, max_reps=1)
    for _ in range(args.warmup):
        _oracle_step(sample)
    times = [_oracle_step(sample) for _ in range(args.steps)]
    t = statistics.mean(times)
    gbs = wl.roofline_bytes(sample) / t / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, args),
        "seq_tokens_per_s": sample.batch / t,
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "note": f"fp64 CPU oracle; full-batch step bytes {nbytes_full}",
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def measure_decode(args, name, dev, dist, rank, world, baseline=True):
    """Time K decode steps of workload `name` (the step --step selects) and
    return the fields of its JSON record (device-timed value and roofline,
    e2e, and on rank 0 of a one-GPU run the CPU baseline and parity)."""
    import torch
    from paged_kv_cache_334_b200 import pa

    w = wl.make_workload(name, seed=rank_seed(args.seed, rank), batch=args.batch,
                         block_size=args.block_size)

    def dev_t(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        if a.dtype == np.uint16:
            t = t.view(torch.bfloat16)
        elif a.dtype == np.uint8:  # E4M3 codes
            t = t.view(torch.float8_e4m3fn)
        return t.to(dev)

    q, kc, vc = dev_t(w.q), dev_t(w.key_cache), dev_t(w.value_cache)
    bt = torch.from_numpy(w.block_tables).to(dev)
    cl = torch.from_numpy(w.context_lens).to(dev)
    has_new = w.slot_mapping is not None
    kn = dev_t(w.k_new) if has_new else None
    vn = dev_t(w.v_new) if has_new else None
    sm = torch.from_numpy(w.slot_mapping).to(dev) if has_new else None
    out = torch.empty_like(q)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    sc = dict(k_scale=w.k_scale, v_scale=w.v_scale)  # FP8 pages: code * scale
    ws = pa.decode_workspace(kc, w.batch, w.num_q_heads, w.max_blocks, **sc)
    scale = 1.0 / math.sqrt(w.head_dim)
    stream = torch.cuda.current_stream(dev)

    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=dev)
    flush_f32 = flush_buf.view(torch.float32)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)
    fused = has_new and args.step == "fused"
    prefix = args.step == "prefix"
    splitk = args.step == "splitk"
    if prefix and not w.shared_prefix_blocks:
        raise SystemExit(f"--step prefix needs a workload with a shared prefix, not {w.name}")
    if splitk:
        P = args.partition_tokens
        maxp = -(-w.max_blocks * w.block_size // P)
        pm = torch.empty(w.batch, w.num_q_heads, maxp, dtype=torch.float32, device=dev)
        ps = torch.empty_like(pm)
        po = torch.empty(w.batch, w.num_q_heads, maxp, w.head_dim, dtype=torch.float32,
                         device=dev)
    # libpa kernels per step.  Groups of 64 or 128 query heads (tensor-core
    # path): the write (inside pa_forward_decode or as its own call), the
    # tile kernel, and its finishing pass or, with a shared prefix, the
    # prefix kernel.  Other groups: the persistent decode kernel and its
    # merge kernel (split-K: pa_reduce's kernel instead), plus the write
    # kernel when the write is a separate call, plus the prefix kernel of
    # the shared-prefix path.
    tensor = tensor_path(w) and not splitk
    if tensor:
        launches_per_step = 2 + (1 if has_new else 0)
    else:
        launches_per_step = 2 + (1 if has_new and not fused else 0) + (1 if prefix else 0)

    def flush_l2():
        # Write a buffer twice the L2 size, then read it back: the step's
        # inputs are evicted and L2 is left holding clean lines, so the timed
        # step pays no write-back of the flush itself.
        flush_buf.zero_()
        torch.amax(flush_f32, out=flush_sink)

    def write():
        if has_new and not fused:
            pa.pa_write_kv_cache(kc, vc, kn, vn, sm, err_word=err, stream=stream, **sc)

    def decode():
        if prefix:
            pa.pa_decode_shared_prefix(out, q, kc, vc, bt, cl, w.shared_prefix_blocks, scale=scale,
                                       err_word=err, stream=stream, **sc)
        elif splitk:
            pa.pa_decode_splitk(q, kc, vc, bt, cl, P, pm, ps, po, scale=scale, err_word=err,
                                stream=stream, **sc)
            pa.pa_reduce(out, pm, ps, po, cl, P, err_word=err, stream=stream)
        elif fused:
            pa.pa_forward_decode(out, q, kc, vc, kn, vn, sm, bt, cl, scale=scale, workspace=ws,
                                 err_word=err, stream=stream, **sc)
        else:
            pa.pa_decode(out, q, kc, vc, bt, cl, scale=scale, workspace=ws, err_word=err,
                         stream=stream, **sc)

    for _ in range(max(args.warmup, 3)):
        flush_l2()
        write()
        decode()
    torch.cuda.synchronize(dev)
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item())} during warm-up")

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    clocks = ClockSampler(dev.index)
    clocks.start()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.mark("t0")
    host_runway()
    for k in range(K):
        flush_l2()
        ev[k][0].record(stream)
        if not fused:
            write()
            ev[k][1].record(stream)
        decode()
        ev[k][2].record(stream)
    torch.cuda.synchronize(dev)
    clocks.mark("t1")
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    step_ms = [e[0].elapsed_time(e[2]) for e in ev]
    # the timed kernel call: pa_forward_decode (the whole step) or the decode
    # call(s) after the write
    dec_ms = step_ms if fused else [e[1].elapsed_time(e[2]) for e in ev]
    t_step = statistics.mean(step_ms)
    t_dec = statistics.mean(dec_ms)

    # end to end: inputs of the step from pinned host memory, output back
    e2e = None
    if not args.no_e2e:
        # the step's inputs (q, tables, lengths, new rows and their slots)
        # staged in one pinned buffer: one host-to-device copy per step, the
        # calls made on views of the device copy
        ins = [q, bt, cl] + ([kn, vn, sm] if has_new else [])
        dev_in, host_in, views = staged_inputs(ins, dev)
        q, bt, cl = views[0], views[1], views[2]
        if has_new:
            kn, vn, sm = views[3], views[4], views[5]
        out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = host_in.numel()
        d2h = out_host.numel() * out_host.element_size()
        Ke = max(3, min(K, 500))
        eve = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(Ke)]
        host_runway()
        for k in range(Ke + 3):
            flush_l2()
            if k >= 3:
                eve[k - 3][0].record(stream)
            dev_in.copy_(host_in, non_blocking=True)
            write()
            decode()
            out_host.copy_(out, non_blocking=True)
            if k >= 3:
                eve[k - 3][1].record(stream)
        torch.cuda.synchronize(dev)
        t_e2e = statistics.mean(e[0].elapsed_time(e[1]) for e in eve)
        e2e = (t_e2e, h2d, d2h)

    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item())}")

    step_bytes = wl.roofline_bytes(w, include_write=has_new)
    dec_bytes = step_bytes if fused else wl.roofline_bytes(w, include_write=False)
    t_step_max = reduce_scalar(t_step, "max", dist, dev)
    bytes_all = reduce_scalar(step_bytes, "sum", dist, dev)
    seqs_all = reduce_scalar(w.batch, "sum", dist, dev)
    ctx_all = reduce_scalar(float(w.context_lens.sum()), "sum", dist, dev)
    e2e_line = None
    if e2e is not None:
        t_e2e_max = reduce_scalar(e2e[0], "max", dist, dev)
        e2e_line = {"value": bytes_all / (t_e2e_max * 1e-3) / 1e9, "unit": "GB/s",
                    "h2d_bytes_per_step": int(e2e[1]), "d2h_bytes_per_step": int(e2e[2]),
                    "ms_per_step": t_e2e_max}

    cpu = parity = None
    if rank == 0 and world == 1:
        if baseline and not args.no_cpu_baseline:
            cpu = cpu_baseline(w, args.cpu_seconds)
        # the timed call's output rows of the first sequences against the oracle
        pidx = parity_indices(w.batch)
        parity = parity_sample(w, out[pidx].double().cpu().numpy(), pidx)

    peak, peak_src = hbm_peak()
    achieved = dec_bytes / (t_dec * 1e-3) / 1e9
    kernel = ("pa_decode_shared_prefix" if prefix else
              "pa_decode_splitk + pa_reduce" if splitk else
              "pa_forward_decode" if fused else "pa_decode")
    roofline_tensor = None
    if prefix or tensor:
        # 64 or 128 query heads per KV head (32 or 64 flop per byte of KV),
        # and a shared prefix, make the call a contraction: its roofline is
        # the tensor-core peak
        tpeak, tpeak_src = tensor_peak()
        tach = attention_flops(w) / (t_dec * 1e-3) / 1e12
        roofline_tensor = {
            "bound": "tensor", "achieved": tach, "peak": tpeak, "unit": "TFLOP/s",
            "frac": tach / tpeak, "traffic": None, "kernel": kernel,
            "flops_per_launch": attention_flops(w), "launch_us": t_dec * 1e3,
            "peak_source": tpeak_src, "hbm_gbs": achieved, "hbm_frac": achieved / peak,
            "ceilings": ceilings(w, attention_flops(w), dec_bytes, t_dec * 1e3,
                                 (clk or {}).get("sm_mhz") or 1965.0),
        }
    traffic = None
    if args.block_size is None and args.batch is None and not prefix:
        traffic = recorded_traffic(name + ("/splitk" if splitk else ""))
    config = workload_config(w, args)
    config["timing"] = RUNWAY_NOTE
    if splitk:
        config["partitions"] = {"tokens": P, "max_partitions": maxp,
                                "partials_bytes": int(pm.numel() * 8 + po.numel() * 4)}
    return {
        "metric": METRIC,
        "value": bytes_all / (t_step_max * 1e-3) / 1e9,
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": t_step_max,
        "step_ms": timing_stats(step_ms),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic",
        "config": config,
        "seq_tokens_per_s": seqs_all / (t_step_max * 1e-3),
        "context_tokens_per_s": ctx_all / (t_step_max * 1e-3),
        "hbm_frac_step": (bytes_all / (t_step_max * 1e-3) / 1e9) / (peak * world),
        "roofline": roofline_tensor if roofline_tensor is not None else {
            "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "traffic": traffic, "kernel": kernel,
            "algorithmic_bytes_per_launch": dec_bytes,
            "launch_us": t_dec * 1e3, "peak_source": peak_src,
        },
        "e2e": e2e_line,
        "cpu_baseline": cpu,
        "parity": parity,
        "gpu_launches": launches_per_step * K,
        "clocks": clk,
    }


def run_ours(args):
    import torch
    from paged_kv_cache_334_b200 import pa

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist(world, local)
    pa.load()

    line = measure_decode(args, args.workload, dev, dist, rank, world)
    if (args.companion != "none" and args.companion != args.workload
            and args.step in ("fused", "separate")):
        # the second configuration the target names, timed the same way in
        # the same run (its own warm-up, K steps, L2 flushes and clocks)
        torch.cuda.empty_cache()
        sub = measure_decode(args, args.companion, dev, dist, rank, world, baseline=False)
        line["gpu_launches"] += sub["gpu_launches"]
        line[args.companion] = {k: sub[k] for k in (
            "value", "unit", "ms_per_step", "step_ms", "hbm_frac_step", "seq_tokens_per_s",
            "context_tokens_per_s", "roofline", "e2e", "parity", "gpu_launches", "clocks",
            "config", "dtype")}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------------------
# --step prefill: one pa_prefill call per step
# ---------------------------------------------------------------------------

PREFILL_METRIC = "paged prefill attention (causal) TFLOP/s and fraction of the B200 bf16 peak"


def prefill_sample(pw, m: int):
    """The oracle's share of a prefill step: sequence 0's last m chunk tokens
    (the same positions, so the same rows of the result)."""
    import dataclasses
    base = pw.base
    n0 = int(pw.chunk_lens[0])
    m = max(1, min(m, n0))
    b1 = dataclasses.replace(base, batch=1, q=base.q[:1].copy(),
                             block_tables=base.block_tables[:1].copy(),
                             context_lens=base.context_lens[:1].copy())
    q = pw.q[n0 - m:n0].copy()
    return wl.PrefillWorkload(base=b1, q=q, query_start=np.array([0, m], dtype=np.int32),
                              chunk_lens=np.array([m], dtype=np.int32),
                              description=f"sequence 0's last {m} of {n0} chunk tokens")


def time_oracle_prefill(pw, target_seconds: float):
    """Time the fp64 oracle's prefill on a sample growing by 4x until one
    pass takes about a quarter of target_seconds, then repeat it to about
    target_seconds."""
    import oracle
    oracle.build()

    def one(s):
        b = s.base
        t0 = time.perf_counter()
        oracle.prefill(s.q, b.key_cache, b.value_cache, b.block_tables, b.context_lens,
                       s.query_start, 1.0 / math.sqrt(b.head_dim))
        return time.perf_counter() - t0

    m = 4
    sample = prefill_sample(pw, m)
    t = one(sample)
    while t < target_seconds / 4 and m < int(pw.chunk_lens[0]):
        m *= 4
        sample = prefill_sample(pw, m)
        t = one(sample)
    total, reps = t, 1
    while total < target_seconds:
        total += one(sample)
        reps += 1
    # the oracle's prefill loops over rows on one thread
    return total / reps, sample, 1, f"{sample.description}, {reps} repetition(s)"


def prefill_parity(pw, sample, out_rows: np.ndarray) -> dict:
    """Max / mean absolute difference between the call's output rows of the
    oracle's sample (sequence 0's last m chunk rows; out_rows holds the
    whole call's rows as float64) and the oracle's prefill of that sample."""
    import oracle
    b = sample.base
    ref, flags = oracle.prefill(sample.q, b.key_cache, b.value_cache, b.block_tables,
                                b.context_lens, sample.query_start, 1.0 / math.sqrt(b.head_dim))
    n0, m = int(pw.chunk_lens[0]), int(sample.chunk_lens[0])
    err = np.abs(np.asarray(out_rows[n0 - m:n0], dtype=np.float64) - ref)
    ok = bool(np.isfinite(err).all()) and not flags.any() and err.max() <= 2e-2 and \
        err.mean() <= 1e-2
    return {"max_abs": float(err.max()), "mean_abs": float(err.mean()), "rows": m,
            "tolerance": {"max_abs": 2e-2, "mean_abs": 1e-2}, "within": bool(ok)}


def run_prefill(args):
    import torch
    from paged_kv_cache_334_b200 import pa

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist(world, local)
    pa.load()

    w = wl.make_workload(args.workload, seed=rank_seed(args.seed, rank),
                         block_size=args.block_size)
    pw = wl.prefill_workload(w, chunk=args.chunk, seed=rank_seed(args.seed, rank))
    base = pw.base

    def dev_t(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return (t.view(torch.bfloat16) if a.dtype == np.uint16 else t).to(dev)

    q, kc, vc = dev_t(pw.q), dev_t(base.key_cache), dev_t(base.value_cache)
    bt, cl, qs = dev_t(base.block_tables), dev_t(base.context_lens), dev_t(pw.query_start)
    out = torch.empty_like(q)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    scale = 1.0 / math.sqrt(base.head_dim)
    mql = pw.max_query_len
    stream = torch.cuda.current_stream(dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=dev)
    flush_f32 = flush_buf.view(torch.float32)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2():
        flush_buf.zero_()
        torch.amax(flush_f32, out=flush_sink)

    def call():
        pa.pa_prefill(out, q, kc, vc, bt, cl, qs, max_query_len=mql, scale=scale,
                      err_word=err, stream=stream)

    for _ in range(max(args.warmup, 3)):
        flush_l2()
        call()
    torch.cuda.synchronize(dev)
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item())} during warm-up")

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    clocks = ClockSampler(local)
    clocks.start()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.mark("t0")
    host_runway()
    for k in range(K):
        flush_l2()
        ev[k][0].record(stream)
        call()
        ev[k][1].record(stream)
    torch.cuda.synchronize(dev)
    clocks.mark("t1")
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    t_call = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)

    e2e = None
    if not args.no_e2e:
        dev_in, host_in, views = staged_inputs([q, bt, cl, qs], dev)
        q, bt, cl, qs = views
        out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = host_in.numel()
        d2h = out_host.numel() * out_host.element_size()
        Ke = max(3, min(K, 200))
        eve = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(Ke)]
        host_runway()
        for k in range(Ke + 3):
            flush_l2()
            if k >= 3:
                eve[k - 3][0].record(stream)
            dev_in.copy_(host_in, non_blocking=True)
            call()
            out_host.copy_(out, non_blocking=True)
            if k >= 3:
                eve[k - 3][1].record(stream)
        torch.cuda.synchronize(dev)
        e2e = (statistics.mean(e[0].elapsed_time(e[1]) for e in eve), h2d, d2h)
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item())}")

    flops = wl.prefill_flops(pw)
    t_max = reduce_scalar(t_call, "max", dist, dev)
    flops_all = reduce_scalar(flops, "sum", dist, dev)
    tokens_all = reduce_scalar(pw.num_tokens, "sum", dist, dev)
    e2e_line = None
    if e2e is not None:
        t_e2e_max = reduce_scalar(e2e[0], "max", dist, dev)
        e2e_line = {"value": flops_all / (t_e2e_max * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": int(e2e[1]), "d2h_bytes_per_step": int(e2e[2]),
                    "ms_per_step": t_e2e_max}
    cpu = parity = None
    if rank == 0 and world == 1:
        rows0 = out[:int(pw.chunk_lens[0])].double().cpu().numpy()
        if args.no_cpu_baseline:
            # the call's last rows of sequence 0 against the oracle, untimed
            sample = prefill_sample(pw, 16)
        else:
            per_step, sample, cores, desc = time_oracle_prefill(pw, args.cpu_seconds)
            cpu = {"value": wl.prefill_flops(sample) / per_step / 1e12, "unit": "TFLOP/s",
                   "cores": cores, "kind": "oracle", "sample": desc,
                   "ms_per_step": per_step * 1e3}
        parity = prefill_parity(pw, sample, rows0)
    tpeak, tpeak_src = tensor_peak()
    hpeak, _ = hbm_peak()
    achieved = flops / (t_call * 1e-3) / 1e12
    nbytes = wl.prefill_roofline_bytes(pw)
    line = {
        "metric": PREFILL_METRIC,
        "value": flops_all / (t_max * 1e-3) / 1e12,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": t_max,
        "step_ms": timing_stats(e[0].elapsed_time(e[1]) for e in ev),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": f"{args.workload} as prefill: {pw.description}",
            "batch": base.batch, "num_q_heads": base.num_q_heads,
            "num_kv_heads": base.num_kv_heads, "head_dim": base.head_dim,
            "block_size": base.block_size, "query_tokens": pw.num_tokens,
            "max_query_len": mql, "context_tokens": int(base.context_lens.sum()),
            "seed": args.seed, "step": "pa_prefill (causal, K/V through the block table)",
            "l2": "flushed before every timed step (zero-fill then read of 2x L2, outside "
                  "the events)",
            "timing": RUNWAY_NOTE,
            "parallelism": f"replicas: one independent batch per GPU x{args.gpus}",
        },
        "query_tokens_per_s": tokens_all / (t_max * 1e-3),
        "roofline": {
            "bound": "tensor", "achieved": achieved, "peak": tpeak, "unit": "TFLOP/s",
            "frac": achieved / tpeak, "traffic": None, "kernel": "pa_prefill",
            "flops_per_launch": flops, "launch_us": t_call * 1e3, "peak_source": tpeak_src,
            "algorithmic_bytes_per_launch": nbytes,
            "hbm_frac": nbytes / (t_call * 1e-3) / 1e9 / hpeak,
        },
        "e2e": e2e_line,
        "cpu_baseline": cpu,
        "parity": parity,
        "gpu_launches": K,
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.step == "prefill":
        if args.impl == "reference":
            raise SystemExit("--step prefill has no reference arm; its cpu_baseline is the "
                             "oracle")
        return run_prefill(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
