"""The multi-GPU path of bench.py on CPU: two gloo ranks, each with its own independent layer
(the path shards by head/layer, so there is no data-path collective), reduce their device
times to the maximum and their work to the sum, exactly as the NCCL run does."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms = [3.0, 5.0][rank]
    flops = [10.0, 20.0][rank]
    t, f = bench.reduce_over_ranks(ms, flops, torch.device("cpu"))
    out[rank] = (t, f)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_reduction_gloo():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    assert out[0] == (5.0, 30.0) and out[1] == (5.0, 30.0)


def test_single_process_is_identity():
    import bench
    assert bench.reduce_over_ranks(2.5, 7.0, torch.device("cpu")) == (2.5, 7.0)
