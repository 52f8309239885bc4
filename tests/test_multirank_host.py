"""Host logic of the multi-rank bench on CPU ranks (gloo, world size 2).

The decode path shards as independent replicas (one per GPU, weak scaling): each rank
builds its own seeded workload and the job's time is the slowest rank's.  These tests
run that logic on two CPU processes; no GPU is involved."""
import os
import socket
import sys
from datetime import timedelta

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        import synth

        vals = bench.max_over_ranks([rank + 1.0, 10.0 - rank, 3.5], "cpu")
        w = bench.replica_workload(synth.WORKLOADS["tiny_h1_n256"], rank)
        k = synth.prefill_layer(w, 0, device="cpu")["K"][1]
        out.put((rank, vals, w.seed, float(k.float().sum())))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_independent_replicas():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in procs:
        rank, vals, seed, ksum = out.get(timeout=120)
        res[rank] = (vals, seed, ksum)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # every rank sees the element-wise maximum
    assert res[0][0] == res[1][0] == [2.0, 10.0, 3.5]
    # replicas: distinct seeds and distinct data, same shapes
    assert res[0][1] != res[1][1]
    assert res[0][2] != res[1][2]


def test_max_over_ranks_single_process():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks([1.0, 2.0], "cpu") == [1.0, 2.0]
