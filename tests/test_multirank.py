"""The bench's multi-rank plumbing on CPU: two gloo ranks (one process per
GPU on a GPU machine) reduce their timings by max and their FLOPs by sum, and each
rank runs its own independently seeded layer (weak scaling, no data-path
collective)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from learned_block_sparse_seer_b200 import synth
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        dev = torch.device("cpu")
        ms = 10.0 + 5.0 * rank          # the slowest rank is the last
        flops = 1e12 * (rank + 1)
        t_max = bench.reduce_over_ranks(ms, dev, "max")
        f_sum = bench.reduce_over_ranks(flops, dev, "sum")
        w = bench.rank_workload(synth.WORKLOADS["tiny"], rank)
        Q, _, _ = synth.make_qkv(w)
        out[rank] = (t_max, f_sum, bench.whole_job_tflops(f_sum, t_max), w.seed, float(Q.sum()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_and_shard():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    r0, r1 = out[0], out[1]
    # both ranks see the max time and the summed FLOPs
    assert r0[0] == r1[0] == 15.0
    assert r0[1] == r1[1] == 3e12
    assert r0[2] == pytest.approx(3e12 / 15e-3 / 1e12)
    # each rank its own layer: distinct seeds and inputs
    assert r0[3] != r1[3] and r0[4] != r1[4]


def test_single_process_reduction_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_over_ranks(7.5, torch.device("cpu"), "max") == 7.5
    assert bench.whole_job_tflops(2e12, 1.0) == pytest.approx(2000.0)
