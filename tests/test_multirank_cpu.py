"""Multi-rank host logic of the benchmark, on CPU with 2 gloo ranks.

The path shards with no exchange step (each rank runs its own independent
batch), so the only cross-rank logic is the timing plumbing: per-rank seeds,
the MAX reduction of the device times (the slowest rank sets the time), and
the whole-job throughput.  Also checks that the reference arm's non-zero ranks
exit without work.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from causal_attention_fwd_b200.synthetic import WORKLOAD_SEED, WORKLOADS, make_inputs

        w = WORKLOADS["tiny"]
        seed = bench.rank_seed(WORKLOAD_SEED[w.name], rank)
        qh, _, _, _ = make_inputs(w.B, w.Hq, w.Hkv, w.S, w.D, seed)
        # rank r pretends its steps took (r + 1) * 10 ms and its stages r-dependent times
        local = [10.0 * (rank + 1), 1.0 + rank, 5.0 - rank, 3.0, 0.5]
        red = bench.reduce_max(local, world)
        tf = bench.whole_job_tflops(w.fwd_flops + w.bwd_flops, 7, red[0], world)
        rc = bench.run_reference(type("A", (), {"workload": "tiny", "steps": 1, "warmup": 0})(), rank,
                                 world) if rank != 0 else None
        q.put((rank, seed, float(qh.float().sum()), red, tf, rc))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, s0, sum0, red0, tf0, _), (r1, s1, sum1, red1, tf1, rc1) = res
    assert s0 != s1 and sum0 != sum1                       # independent batches
    assert red0 == red1 == [20.0, 2.0, 5.0, 3.0, 0.5]      # max over ranks, same on both
    from causal_attention_fwd_b200.synthetic import WORKLOADS

    w = WORKLOADS["tiny"]
    expect = 2 * (w.fwd_flops + w.bwd_flops) * 7 / 20e-3 / 1e12
    assert tf0 == pytest.approx(expect) and tf1 == pytest.approx(expect)
    assert rc1 == 0                                        # reference arm: rank 1 does nothing


def test_single_rank_reduce_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.reduce_max([1.5, 2.0], 1) == [1.5, 2.0]
    assert bench.whole_job_tflops(1e12, 1, 1000.0, 1) == pytest.approx(1.0)
