"""The multi-GPU path is replicas only: the host-side logic (per-rank seeds, max-over-ranks timing, whole-job
throughput) runs here as two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_diffusion_moe_dllm_b200 import replicas


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    w, r, l = replicas.env()
    assert (w, r, l) == (world, rank, rank)
    local = 0.5 + rank            # rank 1 is the slow one
    slow = replicas.max_over_ranks(local, "cpu")
    out[rank] = (slow, replicas.replica_seed(7, rank), replicas.aggregate_throughput(100.0, slow, world))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 1.5                 # both ranks see the slowest time
    assert res[0][1] != res[1][1]                        # replicas draw different requests
    assert res[0][2] == res[1][2] == pytest.approx(200.0 / 1.5)


def test_single_process_without_group():
    assert replicas.max_over_ranks(0.25, "cpu") == 0.25
    assert replicas.env()[0] >= 1
