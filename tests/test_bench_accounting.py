"""The benchmark's work accounting (the numerator of every TFLOPS figure it prints), checked on
CPU tensors against the oracle: selected FLOPs over valid tokens, token-exact frame FLOPs from
the entry codes, the MMA FLOPs of the 128-row tiles, and the router's algorithmic bytes."""
import math

import numpy as np
import torch

import bench
import oracle


class _Csr:
    """The fields of the library's CSR buffers that the accounting reads, on the CPU."""

    def __init__(self, mask, codes=None):
        BH, nb, _ = mask.shape
        rp, ci = oracle.csr_from_mask(mask)
        self.nb = nb
        self.row_ptr = torch.from_numpy(rp.astype(np.int32))
        self.col_idx = torch.from_numpy(ci.astype(np.int32))
        self.nnz = torch.tensor([len(ci)], dtype=torch.int64)
        self.tile_cost = torch.from_numpy(oracle.tile_costs(mask).reshape(-1).astype(np.int32))
        self.col_code = None if codes is None else torch.from_numpy(np.asarray(codes, dtype=np.int32))


def test_selected_flops_and_tile_flops_match_the_oracle():
    rng = np.random.default_rng(0)
    for S, BH, d in ((1000, 3, 128), (64 * 9, 2, 64), (40, 1, 128)):
        nb = -(-S // 64)
        mask = rng.random((BH, nb, nb)) < 0.3
        mask[:, np.arange(nb), np.arange(nb)] = True
        csr = _Csr(mask)
        flops, nnz, padded, kv = bench.selected_flops_from_csr(csr, S, d)
        assert flops == oracle.selected_flops(mask, S, 64, d)
        assert nnz == int(mask.sum()) and padded == 4 * d * 64 * 64 * nnz
        n = np.array([min(S, (j + 1) * 64) - j * 64 for j in range(nb)])
        assert kv == int((mask * n[None, None, :]).sum())
        assert bench.tile_mma_flops(csr, d) == 4 * d * 128 * 64 * int(oracle.tile_costs(mask).sum())


def test_token_exact_flops_count_the_token_mask():
    # entry codes from the oracle; the count must equal the allowed token pairs of the dense mask
    rng = np.random.default_rng(1)
    S, d, fl = 1800, 16, 200
    Q, K = rng.standard_normal((2, S, d)), rng.standard_normal((2, S, d))
    cfg = oracle.RouteCfg(mode="frame_topk", frame_len=fl, topk_frames=2, force_diag=True, frame_exact=True)
    r = oracle.route(Q, K, cfg)
    bf = oracle.block_forced(S, cfg)
    rp, ci = oracle.csr_from_mask(r["mask"])
    nb = r["nb"]
    codes = [oracle.frame_entry_code(r["frame_sets"][row // nb], bf, row % nb, int(ci[e]), S, cfg)
             for row in range(2 * nb) for e in range(rp[row], rp[row + 1])]
    csr = _Csr(r["mask"], codes)
    pairs = sum(int(oracle.frame_token_mask(r["frame_sets"][bh], S, cfg).sum()) for bh in range(2))
    assert bench.selected_flops_exact(csr, S, d) == 4 * d * pairs


def test_router_bytes():
    # Q and K read once plus the CSR, loads and schedule writes
    BH, S, d, nb, nnz = 40, 32760, 128, 512, 12345
    nt = BH * 256
    want = 2 * BH * S * d * 2 + 4 * (BH * nb + 1) + 4 * nnz + 8 * BH + 8 * nt + 8
    assert bench.router_bytes(BH, S, d, 2, nb, nnz) == want


def test_oracle_baseline_sample_scaling():
    # The oracle baselines scale a timed sample to the layer: the router time by heads and the
    # attention time by selected FLOPs. With every head routed and every query block sampled the
    # scale is 1, so the estimate is the sample's own time; a small layer with fewer query blocks
    # than asked for samples all of them.
    from workloads import get_workload, make_inputs
    w = get_workload("tiny")
    x = make_inputs(w)
    r, layer_flops, t_route = bench.oracle_layer(w, x["q"], x["k"])
    BH = w.B * w.H
    assert layer_flops == oracle.selected_flops(r["mask"], w.S, 64, w.d) > 0
    t_layer, desc = bench.oracle_sample(w, x["q"], x["k"], x["v"], r, layer_flops, n_items=10 ** 6,
                                        route_heads=BH, seed=0, t_route_all=t_route)
    assert t_layer > t_route and f"{BH * w.nb} query blocks" in desc
    t1, d1 = bench.oracle_sample(w, x["q"], x["k"], x["v"], r, layer_flops, n_items=4, route_heads=1, seed=1)
    assert t1 > 0 and "router on 1/2 heads" in d1
