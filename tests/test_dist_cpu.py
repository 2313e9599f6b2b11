"""The N > 1 path of bench.py on CPU: two gloo ranks, replicas only.

The routed path has no exchange step, so ranks share nothing but the barrier
around the timed region and the max of their step times.  Each rank runs its
own seeded batch (same shapes, different draws).
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    import datetime

    import bench
    import gqe_synth

    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(ws)
        # step times differ per rank; every rank must see the slowest one
        step_ms = 10.0 + 5.0 * rank
        mx = bench.max_over_ranks(step_ms, ws)
        w = bench.workload_for_rank(gqe_synth.WORKLOADS["tiny_f32"], rank)
        x = gqe_synth.make_inputs(w)["x"]
        xs = [torch.empty_like(x) for _ in range(ws)]
        dist.all_gather(xs, x)
        same_batch = all(torch.equal(xs[0], xi) for xi in xs[1:])
        value = bench.aggregate_value(work=1e9, ws=ws, steps=4, step_ms_max=mx, scale=1e-9)
        bench.barrier(ws)
        out.put((rank, mx, w.seed, same_batch, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_replicas():
    ws = 2
    ctx = mp.get_context("spawn")
    out = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, ws, port, out)) for r in range(ws)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    res = sorted(out.get() for _ in range(ws))
    base_seed = __import__("gqe_synth").WORKLOADS["tiny_f32"].seed
    for rank, mx, seed, same_batch, value in res:
        assert mx == pytest.approx(15.0)          # max over ranks, not the local time
        assert not same_batch                     # each replica draws its own batch
        # whole-job value: both ranks' 4 steps of 1 GFLOP over the slowest 15 ms
        assert value == pytest.approx(2 * 4 * 1.0 / 15e-3)
    assert res[0][2] == base_seed and res[1][2] != base_seed


def test_aggregate_value_single_rank():
    import bench

    assert bench.aggregate_value(work=2e12, ws=1, steps=10, step_ms_max=20.0, scale=1e-12) == pytest.approx(1000.0)
    assert bench.max_over_ranks(3.5, 1) == 3.5
