"""Runtime load balancing across ranks on CPU process groups (gloo), world sizes 2 and 3.

The exchange of balanced_attention (load all-gather, the plan of fvattn_rlb_plan, point-to-
point Q/K/V migration and the return of the outputs) runs for real; the per-rank compute is the
oracle's routing and attention, injected through the Kernels interface. Every rank's output
must equal the oracle attention of its own heads under its own routing, whatever moved."""
import math
import os
import socket

import numpy as np
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


class OracleKernels:
    def __init__(self, p):
        import oracle
        self.o = oracle
        self.cfg = oracle.RouteCfg(p=p)

    def route(self, q, k):
        return self.o.route(q[0], k[0], self.cfg)

    # the router in two stages: record the pooled block ranges, route on the full heads at the end
    def begin_route(self, q):
        return {"ranges": []}

    def pool_blocks(self, handle, q, k, b0, b1):
        handle["ranges"].append((b0, b1))
        handle["q"], handle["k"] = q, k          # the full heads, filled slice by slice

    def finish_route(self, handle, q):
        nb = -(-q.shape[2] // 64)
        covered = sorted(handle["ranges"])
        assert covered[0][0] == 0 and covered[-1][1] == nb
        assert all(a[1] == b[0] for a, b in zip(covered, covered[1:])), covered
        assert handle["q"] is q
        return self.route(handle["q"], handle["k"])

    def head_load(self, state):
        return torch.from_numpy(self.o.head_loads(state["mask"]))

    def attend(self, q, k, v, state, active, out):
        Hl, S, d = q.shape[1], q.shape[2], q.shape[3]
        items = [(h, i) for h in range(Hl) if active is None or active[h] for i in range(state["nb"])]
        ref = self.o.attention_rows(q[0], k[0], v[0], state["mask"], 1.0 / math.sqrt(d), items)
        for (h, i), rows in ref.items():
            out[0, h, i * 64: i * 64 + rows.shape[0]] = torch.from_numpy(rows).to(out.dtype)


def _inputs(rank):
    from workloads import get_workload, make_inputs
    # rank 0: unclustered tokens (routing keeps most blocks); other ranks: strongly clustered
    alpha = ("const", 0.0) if rank == 0 else ("const", 3.0)
    w = get_workload("tiny", H=3, S=512, alpha=alpha, seed=10 + rank)
    x = make_inputs(w)
    return x["q"], x["k"], x["v"]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from block_sparse_top_fvattn_b200 import rlb
        q, k, v = _inputs(rank)
        kern = OracleKernels(0.9)
        o, plan = rlb.balanced_attention(q, k, v, group=None, target=1.05, max_moves_per_rank=2, kernels=kern)
        ref = torch.empty_like(q)
        kern.attend(q, k, v, kern.route(q, k), None, ref)
        out[rank] = (float((o - ref).abs().max()), plan.moves, plan.imbalance_before, plan.imbalance_after)
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_balanced_attention_gloo(world):
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    moves = out[0][1]
    for r in range(world):
        err, mv, before, after = out[r]
        assert err == 0.0, (r, err)                # a migrated head is computed exactly as at home
        assert mv == moves                         # every rank computed the same plan
    assert len(moves) > 0 and all(s == 0 for s, _, _ in moves[:1])   # the heavy rank sends first
    assert out[0][3] < out[0][2]                  # the imbalance went down


def _ulysses_worker(rank, world, port, balance, overlap, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from block_sparse_top_fvattn_b200 import ulysses
        from workloads import get_workload, make_inputs
        # one global layer (the same draw on every rank), sequence-sharded across the ranks
        w = get_workload("tiny", H=2 * world, S=256 * world, alpha=("uniform", 0.0, 3.0), seed=21)
        x = make_inputs(w)
        Sl = w.S // world
        shard = [t[:, :, rank * Sl:(rank + 1) * Sl].contiguous() for t in (x["q"], x["k"], x["v"])]
        kern = OracleKernels(0.9)
        o, plan = ulysses.ulysses_attention(*shard, group=None, balance=balance, target=1.0, overlap_pool=overlap,
                                            max_moves_per_rank=1, kernels=kern)
        ref = torch.empty_like(x["q"])
        kern.attend(x["q"], x["k"], x["v"], kern.route(x["q"], x["k"]), None, ref)
        out[rank] = float((o - ref[:, :, rank * Sl:(rank + 1) * Sl]).abs().max())
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world,balance,overlap", [(2, False, False), (2, True, False), (3, True, False),
                                                   (2, False, True), (3, True, True)])
def test_ulysses_attention_gloo(world, balance, overlap):
    # sequence -> heads all-to-all, routing and attention of the local heads (with head migration
    # when balance), heads -> sequence: each rank's output slice equals the single-process
    # oracle attention of the whole layer
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_ulysses_worker, args=(world, _free_port(), balance, overlap, out), nprocs=world,
                       start_method="spawn", join=True)
    for r in range(world):
        assert out[r] == 0.0, (r, out[r])
