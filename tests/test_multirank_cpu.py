"""Host logic of the multi-rank benchmark path on CPU: two gloo ranks.

The prefill shards over independent sequences, so ranks never exchange data;
the only collectives are the barrier around the timed region and the max of
the per-rank times.  This runs those helpers of bench.py on world_size 2 with
the gloo backend (no GPU) and checks the reduction, the weak-scaling
aggregate and that every rank draws its own inputs."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    from delta_rule_linear_kla_b200 import inputs

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dev = torch.device("cpu")
        bench.barrier(world)
        ms = 1.0 + rank  # rank 1 is the slow one
        ms_max = bench.allreduce_max(ms, world, dev)
        w = bench.rank_workload(inputs.WORKLOADS["tiny"], rank)
        x = inputs.make_prefill(w)
        value = bench.aggregate_throughput(w.B * w.T, world, ms_max)
        out[rank] = (ms_max, value, float(x["q"].double().sum()), w.seed)
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_weak_scaling():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    (m0, v0, s0, seed0), (m1, v1, s1, seed1) = out[0], out[1]
    assert m0 == m1 == 2.0                       # max over ranks, agreed by both
    assert v0 == v1 == pytest.approx(1 * 256 * 2 / 2e-3)  # all ranks' tokens / slowest time
    assert seed0 != seed1 and s0 != s1           # each rank has its own sequences
