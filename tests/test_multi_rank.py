"""The benchmark's multi-process logic on CPU with the gloo backend.

On the GPU pool every call gets one GPU, so the replica path of
`bench.py --gpus N` (one process per GPU, each with its own token batch, no
collective on the data path) is exercised here with world size 2: the
max-over-ranks reduction of the step time, the barrier, and the per-rank
seed offsets that make each replica's activations different.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist

    import bench
    from i2_mpgemm_b200 import inputs
    r, w = bench.dist_init("gloo")
    assert (r, w) == (rank, world)
    got = bench.max_over_ranks(1.5 + rank, device=torch.device("cpu"))
    bench.barrier()
    x0 = inputs.activations(1, 256, inputs.seed_stack(0, 0) + 7919 * rank)
    out[rank] = (got, float(x0.sum()))
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_replicas_reduce_the_max_time_and_use_distinct_inputs():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(90)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0][0] == res[1][0] == 2.5       # both ranks see the slowest rank's time
    assert res[0][1] != res[1][1]              # replicas draw different token batches


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.dist_env()[1] >= 1
