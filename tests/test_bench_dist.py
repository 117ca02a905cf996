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
