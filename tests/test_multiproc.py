"""The benchmark's multi-rank plumbing on CPU: two gloo ranks on 127.0.0.1,
rendezvous from the torchrun environment variables, barrier, the max over
ranks of the timed seconds, the whole-job throughput of weak scaling, and a
batch of its own per rank (seed + rank).  No GPU and no collective on the data
path: requests are independent, so ranks are replicas."""

import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    # host-side plumbing only: no rank may pick a GPU (on a one-GPU machine the
    # second rank's device would not exist), so gloo is what runs
    os.environ["CUDA_VISIBLE_DEVICES"] = ""
    sys.path.insert(0, ROOT)
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import bench
    import torch.distributed as dist
    r, w, local = bench.dist_setup()
    try:
        assert (r, w, local) == (rank, world, rank)
        bench.barrier(w)
        my_seconds = 1.0 + rank                     # rank 1 is the slow one
        slowest = bench.max_over_ranks(my_seconds, w, "cpu")
        value = bench.job_throughput(1000.0, 10, w, slowest)
        wl = bench.workload_for("llama8b_decode", 0 + rank)
        out.put((rank, slowest, value, [int(x) for x in wl.seq_lens[:4]]))
        bench.barrier(w)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    mp.start_processes(_rank_main, args=(world, port, q), nprocs=world, join=True,
                       start_method="spawn")
    res = sorted(q.get() for _ in range(world))
    for rank, slowest, value, lens in res:
        assert slowest == 2.0                       # max over ranks, on every rank
        assert value == pytest.approx(1000.0 * 10 * 2 / 2.0)
    assert res[0][3] != res[1][3]                   # each rank draws its own batch
