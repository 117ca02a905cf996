"""The multi-GPU host logic of bench.py on CPU: two gloo ranks.

Every rank decodes its own independent, seeded batch (weak scaling) and the
only cross-rank traffic is the timing reduction: max of the step time, sum of
the bytes and sequences.  No data-path collective exists to test."""
import multiprocessing as mp
import os
import socket

import numpy as np


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    from paged_kv_cache_334_b200 import workloads as wl
    w_, r_, l_ = bench.dist_env()
    dist = bench.init_dist(w_, l_, backend="gloo")
    w = wl.make_workload("gqa_bf16", seed=bench.rank_seed(0, r_), batch=4)
    t_step = 1.0 + r_  # rank 1 is the slow one
    mx = bench.reduce_scalar(t_step, "max", dist, "cpu")
    tot = bench.reduce_scalar(wl.roofline_bytes(w), "sum", dist, "cpu")
    seqs = bench.reduce_scalar(w.batch, "sum", dist, "cpu")
    out_q.put((r_, w_, mx, tot, seqs, wl.roofline_bytes(w), w.context_lens.tolist()))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_weak_scaling_reductions():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, mx0, tot0, s0, b0, c0), (r1, w1, mx1, tot1, s1, b1, c1) = res
    assert (r0, r1, w0, w1) == (0, 1, 2, 2)
    assert mx0 == mx1 == 2.0                 # slowest rank's time
    assert tot0 == tot1 == b0 + b1           # bytes of all ranks
    assert s0 == s1 == 8                     # sequences of all ranks
    assert c0 != c1                          # independent batches per rank


def test_rank_zero_alone_runs_the_reference_arm(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0"]) == 0
    assert capsys.readouterr().out == ""     # non-zero ranks exit without work


def test_prefill_step_arguments_and_oracle_sample():
    """--step prefill: its arguments, the refusal of a reference arm, and the
    oracle's sample (sequence 0's last m chunk rows at their own positions)."""
    import pytest

    import bench
    from paged_kv_cache_334_b200 import workloads as wl

    a = bench.parse_args(["--step", "prefill", "--chunk", "64"])
    assert a.step == "prefill" and a.chunk == 64 and a.workload == "gqa_bf16"
    with pytest.raises(SystemExit):
        bench.main(["--step", "prefill", "--impl", "reference"])
    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=3, num_q_heads=8, num_kv_heads=2,
                           head_dim=64, block_size=4, context_lens=[9, 5, 3], seed=1,
                           new_tokens=True)
    pw = wl.prefill_workload(w, chunk=6, seed=1)
    s = bench.prefill_sample(pw, 4)
    assert s.base.batch == 1 and s.query_start.tolist() == [0, 4]
    assert int(s.base.context_lens[0]) == 9 and s.chunk_lens.tolist() == [4]
    assert np.array_equal(s.q, pw.q[2:6])  # chunk rows 2..5 of sequence 0: positions 5..8
    assert bench.prefill_sample(pw, 100).chunk_lens.tolist() == [6]
    # the sample's rows are the full call's rows at those positions
    import oracle
    b = pw.base
    full, _ = oracle.prefill(pw.q, b.key_cache, b.value_cache, b.block_tables, b.context_lens,
                             pw.query_start)
    part, _ = oracle.prefill(s.q, s.base.key_cache, s.base.value_cache, s.base.block_tables,
                             s.base.context_lens, s.query_start)
    assert np.isfinite(full).all() and np.array_equal(part, full[2:6])


def test_cpu_baseline_reports_threads_and_a_single_thread_run():
    """The oracle baseline states the threads its OpenMP loops used, adds a
    one-thread run on a smaller sample, and leaves the thread count as it
    was; the step statistics are mean / median / min / max."""
    import bench
    import oracle
    from paged_kv_cache_334_b200 import workloads as wl

    w = wl.make_workload("gqa_bf16", seed=0, batch=3)
    before = oracle.max_threads()
    line = bench.cpu_baseline(w, 0.2)
    assert oracle.max_threads() == before
    assert line["cores"] == before and line["kind"] == "oracle" and line["value"] > 0
    st = line["single_thread"]
    assert st["cores"] == 1 and st["value"] > 0 and st["ms_per_step"] > 0
    s = bench.timing_stats([3.0, 1.0, 2.0, 10.0])
    assert s == {"mean": 4.0, "median": 2.5, "min": 1.0, "max": 10.0}


def test_ceilings_of_a_tensor_path_call():
    """The three lower bounds of one call (HBM bytes, tensor flops, one ex2
    per score) and the call's time as a fraction of each."""
    import bench
    from paged_kv_cache_334_b200 import workloads as wl

    w = wl.make_workload("mqa_prefix_bf16", seed=0, batch=4)
    flops = bench.attention_flops(w)
    nbytes = wl.roofline_bytes(w, include_write=False)
    c = bench.ceilings(w, flops, nbytes, 50.0, 1965.0)
    exps = float(w.context_lens.sum()) * 64
    assert c["ex2_per_launch"] == exps
    assert abs(c["ex2_us"] - exps / (148 * 16 * 1965e6) * 1e6) < 1e-9
    hbm, _ = bench.hbm_peak()
    tp, _ = bench.tensor_peak()
    assert abs(c["hbm_us"] - nbytes / hbm / 1e3) < 1e-9
    assert abs(c["tensor_us"] - flops / tp / 1e6) < 1e-9
    for k in ("hbm", "tensor", "ex2"):
        assert abs(c[k + "_frac"] - c[k + "_us"] / 50.0) < 1e-12


def test_parity_sample_against_the_oracle():
    """bench's parity record: zero against the oracle's own rows, the size
    of a planted error otherwise, and the dtype's tolerance."""
    import math

    import bench
    import oracle
    from paged_kv_cache_334_b200 import workloads as wl

    for name in ("gqa_bf16", "gqa_fp8"):
        w = wl.make_workload(name, seed=2, batch=3)
        kc, vc = w.key_cache.copy(), w.value_cache.copy()
        if name == "gqa_fp8":
            oracle.write_kv_cache_fp8(kc, vc, w.k_new, w.v_new, w.slot_mapping, w.k_scale,
                                      w.v_scale)
            ref, _ = oracle.decode_fp8(w.q, kc, vc, w.k_scale, w.v_scale, w.block_tables,
                                       w.context_lens, 1.0 / math.sqrt(w.head_dim))
        else:
            oracle.write_kv_cache(kc, vc, w.k_new, w.v_new, w.slot_mapping)
            ref, _ = oracle.decode(w.q, kc, vc, w.block_tables, w.context_lens,
                                   1.0 / math.sqrt(w.head_dim))
        idx = bench.parity_indices(w.batch)
        assert idx == [0, 1, 2]
        rec = bench.parity_sample(w, ref[idx], idx)
        assert rec["max_abs"] == 0.0 and rec["within"] and rec["sequences"] == idx
        # rows of any subset, in the subset's order
        rec = bench.parity_sample(w, ref[[2, 0]], [2, 0])
        assert rec["max_abs"] == 0.0 and rec["within"]
        bad = ref.copy()
        bad[1, 3, 5] += 0.05
        rec = bench.parity_sample(w, bad[idx], idx)
        assert abs(rec["max_abs"] - 0.05) < 1e-12 and not rec["within"]
        assert rec["tolerance"] == {"max_abs": 2e-2, "mean_abs": 1e-2}
    # spread over a large batch, ends included
    idx = bench.parity_indices(128)
    assert idx[0] == 0 and idx[-1] == 127 and len(idx) == 12


def test_prefill_parity_record():
    import bench
    import oracle
    from paged_kv_cache_334_b200 import workloads as wl

    w = wl.custom_workload(dtype=wl.DTYPE_BF16, batch=2, num_q_heads=8, num_kv_heads=2,
                           head_dim=64, block_size=4, context_lens=[9, 5], seed=4,
                           new_tokens=True)
    pw = wl.prefill_workload(w, seed=4)
    b = pw.base
    full, _ = oracle.prefill(pw.q, b.key_cache, b.value_cache, b.block_tables, b.context_lens,
                             pw.query_start)
    s = bench.prefill_sample(pw, 3)
    rec = bench.prefill_parity(pw, s, full)
    assert rec["max_abs"] == 0.0 and rec["within"] and rec["rows"] == 3
    bad = full.copy()
    bad[7, 0, 0] += 0.5  # a row of the sample (sequence 0's rows 6..8)
    assert not bench.prefill_parity(pw, s, bad)["within"]
    bad = full.copy()
    bad[2, 0, 0] += 0.5  # outside the sample
    assert bench.prefill_parity(pw, s, bad)["within"]


def test_staged_inputs_pack_a_step_into_one_copy(monkeypatch):
    """The e2e loop's staging: every input lands in one buffer, 256-byte
    aligned, and the device views equal the tensors they stand for."""
    import torch

    import bench
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)  # no device here
    a = torch.arange(10, dtype=torch.int32)
    b = torch.randn(3, 4).to(torch.bfloat16)
    c = torch.arange(5, dtype=torch.int64)
    dev_buf, host_buf, views = bench.staged_inputs([a, b, c], torch.device("cpu"))
    assert torch.equal(views[0], a) and torch.equal(views[2], c)
    assert torch.equal(views[1].view(torch.int16), b.view(torch.int16))
    assert torch.equal(dev_buf, host_buf) and dev_buf.numel() == 3 * 256
    for v in views:
        assert (v.data_ptr() - dev_buf.data_ptr()) % 256 == 0


def test_recorded_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    """roofline.traffic comes from the row of the current kernel sources
    only: a row under another hash, or no row, gives None."""
    import bench
    h = bench.decode_source_hash()
    f = tmp_path / "traffic.md"
    f.write_text("| workload | source hash | dram bytes per call |\n|---|---|---|\n"
                 f"| gqa_bf16 | {h} | 123456 |\n"
                 "| mixed_bf16 | 0000000000000000 | 999 |\n"
                 f"| long_bf16/splitk | {h} | 777 |\n")
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.recorded_traffic("gqa_bf16") == 123456.0
    assert bench.recorded_traffic("long_bf16/splitk") == 777.0
    assert bench.recorded_traffic("mixed_bf16") is None      # another hash
    assert bench.recorded_traffic("gqa_fp8") is None         # no row
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "absent.md"))
    assert bench.recorded_traffic("gqa_bf16") is None
