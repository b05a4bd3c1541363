"""GPU side of runtime load balancing: fvattn_select_heads restricts the attention to a subset
of heads (the heads a rank keeps), leaves the other heads' output rows untouched and keeps the
longest-first order of the kept tiles; balanced_attention runs end to end on one rank."""
import numpy as np
import pytest
import torch

import block_sparse_top_fvattn_b200 as fv
from test_gpu_parity import compare_attention, compare_csr
from workloads import get_workload, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fv.load()


def _inputs(name, **kw):
    w = get_workload(name, **kw)
    x = make_inputs(w)
    return w, x["q"].cuda(), x["k"].cuda(), x["v"].cuda()


@pytest.mark.parametrize("name,kw,active", [
    ("single", {"H": 4, "S": 2000}, [1, 0, 1, 0]),
    ("single", {"H": 3, "S": 64 * 9 + 7, "d": 64}, [0, 0, 1]),
    ("tiny", {}, [0, 1]),                                   # fp32 path
    ("single", {"H": 2, "S": 1024}, [0, 0]),                # nothing kept
])
def test_select_heads(name, kw, active):
    w, q, k, v = _inputs(name, **kw)
    H = q.shape[1]
    cfg = fv.RouteConfig(p=0.9)
    csr = fv.route(q, k, cfg)
    _, gm, r = compare_csr(csr, q, k, cfg)
    full = fv.sparse_attn(q, k, v, csr).clone()
    assert fv.read_status(csr) == 0
    nt = -(-w.nb // 2)
    assert int(csr.status[3].item()) == H * nt
    order = csr.tile_order.cpu().numpy().copy()
    fv.select_heads(csr, torch.tensor(active, dtype=torch.uint8, device="cuda"))
    out = torch.full_like(q, 7.0)
    fv.sparse_attn(q, k, v, csr, out=out)
    assert fv.read_status(csr) == 0
    kept = [h for h in range(H) if active[h]]
    dropped = [h for h in range(H) if not active[h]]
    n = int(csr.status[3].item())
    assert n == len(kept) * nt
    want = [t for t in order if active[t // nt]]
    np.testing.assert_array_equal(csr.tile_order[:n].cpu().numpy(), np.array(want, dtype=np.int32))
    for h in kept:
        assert torch.equal(out[:, h], full[:, h])           # same kernels, same tiles: bit-identical
    for h in dropped:
        assert bool((out[:, h] == 7.0).all())
    if kept:
        # the kept heads against the oracle's attention (B = 1: head index = bh)
        items = [(h, i) for h in kept for i in range(w.nb)]
        lim = (1e-4, 1e-4) if w.dtype == "f32" else (2e-2, 2e-3)
        compare_attention(out, q, k, v, r, gm, 1.0 / np.sqrt(w.d), items, *lim)
    fv.route(q, k, cfg, csr=csr)                            # routing again selects every head
    torch.cuda.synchronize()
    assert int(csr.status[3].item()) == H * nt


def test_balanced_attention_one_rank_nccl(tmp_path):
    import torch.distributed as dist
    from block_sparse_top_fvattn_b200 import rlb
    w, q, k, v = _inputs("single", H=3, S=1500)
    dist.init_process_group("nccl", init_method=f"file://{tmp_path}/pg", rank=0, world_size=1)
    try:
        out, plan = rlb.balanced_attention(q, k, v, fv.RouteConfig(p=0.9), target=1.0, max_moves_per_rank=1)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert plan.moves == [] and plan.imbalance_before == 1.0
    csr = fv.route(q, k, fv.RouteConfig(p=0.9))
    ref = fv.sparse_attn(q, k, v, csr)
    assert torch.equal(out, ref)
    np.testing.assert_array_equal(plan.loads[0], csr.head_load.cpu().numpy())


@pytest.mark.parametrize("overlap_pool,balance", [(True, True), (False, False)])
def test_ulysses_attention_one_rank_nccl_against_oracle(tmp_path, overlap_pool, balance):
    # The sequence-parallel layer on one NCCL rank: the all-to-alls are identities, the router
    # runs in two stages (pooling the one "arriving" slice, then finishing), and balanced
    # attention plans no move. The output is compared with the oracle's attention under the
    # oracle's own routing, in Top-p mode and in token-exact frame mode.
    import torch.distributed as dist
    import oracle
    from block_sparse_top_fvattn_b200 import ulysses
    w, q, k, v = _inputs("single", H=2, S=64 * 40, frame_len=640, region_len=128)
    cfgs = [fv.RouteConfig(p=0.9),
            fv.RouteConfig(mode="frame_topk", topk_frames=1, frame_len=640, frame_window=0, force_first_frame=True,
                           frame_exact=True)]
    dist.init_process_group("nccl", init_method=f"file://{tmp_path}/pg", rank=0, world_size=1)
    try:
        outs = []
        for cfg in cfgs:
            o, plan = ulysses.ulysses_attention(q, k, v, cfg, balance=balance, target=1.0, overlap_pool=overlap_pool)
            torch.cuda.synchronize()
            outs.append(o)
            if balance:
                assert plan.moves == []
    finally:
        dist.destroy_process_group()
    B, H, S, d = q.shape
    Q, K, V = (t.reshape(B * H, S, d).cpu() for t in (q, k, v))
    for cfg, o in zip(cfgs, outs):
        oc = oracle.RouteCfg(mode=cfg.mode, p=cfg.p, force_diag=cfg.force_diag, frame_len=cfg.frame_len,
                             topk_frames=cfg.topk_frames, frame_window=cfg.frame_window,
                             force_first_frame=cfg.force_first_frame, frame_exact=cfg.frame_exact)
        r = oracle.route(Q, K, oc)
        if cfg.frame_exact:
            tok = np.stack([oracle.frame_token_mask(r["frame_sets"][bh], S, oc) for bh in range(B * H)])
            ref = oracle.attention_dense_mask(Q, K, V, tok, 1.0 / np.sqrt(d))
        else:
            ref = oracle.attention_sets(Q, K, V, r["mask"], 1.0 / np.sqrt(d))
        # query blocks whose selection is a near-tie may legitimately differ: left out
        keep = np.repeat(~r["near_tie"], 64, axis=1)[:, :S]
        assert keep.mean() > 0.9
        e = np.abs(o.reshape(B * H, S, d).float().cpu().numpy() - ref)[keep]
        assert e.max() <= 2e-2 and e.mean() <= 2e-3, (cfg.mode, e.max(), e.mean())


def test_lazy_router_reuses_the_routing():
    # Diffusion steps with new inputs: steps between refreshes attend with the last refresh's
    # selection, exactly as the oracle does with that (stale) mask.
    import oracle
    w = get_workload("single", H=2, S=1100)
    layer = fv.LazyRouter(fv.RouteConfig(p=0.9), refresh_every=3)
    masks = {}
    for step in range(5):
        x = make_inputs(w, seed=100 + step)
        q, k, v = x["q"].cuda(), x["k"].cuda(), x["v"].cuda()
        o = layer(q, k, v, step)
        assert fv.read_status(layer.csr) == 0
        B, H, S, d = q.shape
        if step % 3 == 0:
            masks["cur"] = oracle.route(x["q"].reshape(B * H, S, d), x["k"].reshape(B * H, S, d),
                                        oracle.RouteCfg(p=0.9))
        r = masks["cur"]
        assert not r["near_tie"].any()                         # these seeds have no near-tie rows
        rp, ci = oracle.csr_from_mask(r["mask"])
        np.testing.assert_array_equal(layer.csr.row_ptr.cpu().numpy(), rp)
        np.testing.assert_array_equal(layer.csr.col_idx[: len(ci)].cpu().numpy(), ci)
        ref = oracle.attention_sets(x["q"].reshape(B * H, S, d), x["k"].reshape(B * H, S, d),
                                    x["v"].reshape(B * H, S, d), r["mask"], 1.0 / np.sqrt(d))
        e = np.abs(o.reshape(B * H, S, d).float().cpu().numpy() - ref)
        assert e.max() <= 2e-2 and e.mean() <= 2e-3
    assert layer.routed == 2                                   # steps 0 and 3


def test_select_heads_reports_a_bad_tile_order():
    # The kernel checks every entry against the tile count before using it; a corrupted entry is
    # dropped and reported as FVATTN_ERR_INVALID (-1) in the device status word.
    w, q, k, v = _inputs("single", H=2, S=1000)
    csr = fv.route(q, k, fv.RouteConfig(p=0.9))
    assert fv.read_status(csr) == 0
    n = csr.tile_order.numel()
    csr.tile_order[0] = n + 5
    csr.tile_order[1] = -3
    fv.select_heads(csr, torch.ones(2, dtype=torch.uint8, device="cuda"))
    assert fv.read_status(csr) == -1
    assert int(csr.status[3].item()) == n - 2          # the other tiles are kept
