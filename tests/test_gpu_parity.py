"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle, on a B200.

Block selections must match bit for bit except on near-tie rows (a cumulative mass within
1e-5 of p at the cut, or a probability gap under 1e-6 at the boundary), where the GPU's set
must be a valid selection. Every expected value comes from the oracle on the same inputs: the
attention reference uses the oracle's selection, and query blocks whose GPU selection
(legitimately) differs are left out of that comparison. Attention outputs must be within
max-abs 2e-2 and mean-abs 2e-3 of the oracle for bf16 inputs (fp32 inputs: the notes' own
full-coverage bound, max-abs 1e-4)."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import block_sparse_top_fvattn_b200 as fv
from workloads import get_workload, make_inputs

pytestmark = pytest.mark.gpu

MAX_ABS_BF16, MEAN_ABS_BF16 = 2e-2, 2e-3
MAX_ABS_F32 = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fv.load()


def gpu_mask(csr) -> np.ndarray:
    rp = csr.row_ptr.cpu().numpy().astype(np.int64)
    ci = csr.col_idx.cpu().numpy()
    BH, nb = csr.B * csr.H, csr.nb
    m = np.zeros((BH * nb, nb), dtype=bool)
    for r in range(BH * nb):
        cols = ci[rp[r]:rp[r + 1]]
        assert np.all(np.diff(cols) > 0), "CSR rows must be strictly ascending"
        m[r, cols] = True
    return m.reshape(BH, nb, nb)


def to_oracle_cfg(cfg: fv.RouteConfig) -> oracle.RouteCfg:
    return oracle.RouteCfg(mode=cfg.mode, p=cfg.p, force_diag=cfg.force_diag, local_window=cfg.local_window,
                           frame_len=cfg.frame_len, topk_frames=cfg.topk_frames, frame_window=cfg.frame_window,
                           force_first_frame=cfg.force_first_frame, topk_blocks=cfg.topk_blocks,
                           sasa_coef=cfg.sasa_coef, sasa_trigger=cfg.sasa_trigger, frame_exact=cfg.frame_exact)


def check_bookkeeping_properties(csr, gm):
    """Invariants of the router's bookkeeping on its own selection, in plain NumPy: row offsets
    are the prefix sums of the row counts, head loads their per-head sums, tile costs the sizes
    of the unions of query blocks 2t and 2t+1, and the tile order is by cost, largest first,
    ties by ascending tile id."""
    BH, nb, _ = gm.shape
    counts = gm.reshape(BH * nb, nb).sum(axis=1)
    np.testing.assert_array_equal(csr.row_ptr.cpu().numpy()[1:], np.cumsum(counts))
    np.testing.assert_array_equal(csr.head_load.cpu().numpy(), gm.sum(axis=(1, 2)))
    nt = -(-nb // 2)
    pair = np.zeros((BH, nt, nb), dtype=bool)
    pair[:, :, :] = gm[:, 0::2]
    pair[:, : nb // 2] |= gm[:, 1::2]
    costs = pair.sum(axis=2).reshape(-1)
    np.testing.assert_array_equal(csr.tile_cost.cpu().numpy(), costs)
    order = csr.tile_order.cpu().numpy()
    assert sorted(order.tolist()) == list(range(costs.size))
    key = np.stack([-costs[order], order], axis=1)
    assert all(tuple(key[t]) <= tuple(key[t + 1]) for t in range(len(order) - 1))
    assert int(csr.nnz.item()) == int(counts.sum())


def check_route(q, k, cfg: fv.RouteConfig, csr=None, r=None):
    """Run the GPU router and compare with the oracle. Returns (csr, gpu mask, oracle result).
    Rows may differ only where the oracle flags a near-tie, and there the GPU's set must be a
    valid selection; the bookkeeping equals the oracle's when no row differs, and satisfies its
    invariants on the GPU's own selection in every case."""
    csr = fv.route(q, k, cfg, csr=csr)
    return compare_csr(csr, q, k, cfg, r)


def compare_csr(csr, q, k, cfg: fv.RouteConfig, r=None):
    """The checks of check_route on a CSR the GPU router has already written. In token-exact
    frame mode the per-entry codes must also equal the oracle's."""
    B, H, S, d = q.shape
    assert fv.read_status(csr) == 0
    gm = gpu_mask(csr)
    oc = to_oracle_cfg(cfg)
    if r is None:
        r = oracle.route(q.reshape(B * H, S, d), k.reshape(B * H, S, d), oc)
    om = r["mask"]
    near = r["near_tie"]
    diff_rows = np.any(gm != om, axis=2)
    bad = diff_rows & ~near
    assert not bad.any(), f"{int(bad.sum())} non-tie rows differ, e.g. {np.argwhere(bad)[:5].tolist()}"
    for bh, i in np.argwhere(diff_rows):
        assert oracle.valid_near_tie_set(r, bh, i, gm[bh, i], S, oc), (bh, i)
    if not diff_rows.any():
        rp, ci = oracle.csr_from_mask(om)
        np.testing.assert_array_equal(csr.row_ptr.cpu().numpy(), rp)
        np.testing.assert_array_equal(csr.col_idx[: len(ci)].cpu().numpy(), ci)
        assert int(csr.nnz.item()) == len(ci)
        np.testing.assert_array_equal(csr.head_load.cpu().numpy(), oracle.head_loads(om))
        costs = oracle.tile_costs(om)
        np.testing.assert_array_equal(csr.tile_cost.cpu().numpy(), costs.reshape(-1))
        np.testing.assert_array_equal(csr.tile_order.cpu().numpy(), oracle.lpt_order(costs))
        if cfg.frame_exact:
            nb = -(-S // 64)
            bf = oracle.block_forced(S, oc)
            want = np.array([oracle.frame_entry_code(r["frame_sets"][row // nb], bf, row % nb, int(ci[e]), S, oc)
                             for row in range(B * H * nb) for e in range(rp[row], rp[row + 1])], dtype=np.int64)
            np.testing.assert_array_equal(csr.col_code[: len(ci)].cpu().numpy().astype(np.int64), want)
    check_bookkeeping_properties(csr, gm)
    return csr, gm, r


def check_attention(q, k, v, csr, r, gm, scale, items=None, max_abs=MAX_ABS_BF16, mean_abs=MEAN_ABS_BF16):
    """The library's attention against the oracle's attention under the oracle's selection
    (r["mask"]). Query blocks whose GPU selection differs from the oracle's (near-tie rows,
    validated by check_route) are left out of the element-wise comparison."""
    o = fv.sparse_attn(q, k, v, csr)
    assert fv.read_status(csr) == 0
    return compare_attention(o, q, k, v, r, gm, scale, items, max_abs, mean_abs)


def compare_attention(o, q, k, v, r, gm, scale, items=None, max_abs=MAX_ABS_BF16, mean_abs=MEAN_ABS_BF16):
    """The checks of check_attention on an output the GPU has already written: the rows of
    `items` ((head, query block) pairs) against the oracle's attention under its own selection,
    leaving out query blocks whose GPU selection differs (validated near-ties)."""
    B, H, S, d = q.shape
    nb = -(-S // 64)
    ref_mask = r["mask"]
    differs = np.any(gm != ref_mask, axis=2)
    if items is None:
        items = [(bh, i) for bh in range(B * H) for i in range(nb)]
    items = [(bh, i) for bh, i in items if not differs[bh, i]]
    assert items, "no query block left to compare"
    Q, K, V = (t.reshape(B * H, S, d).cpu() for t in (q, k, v))
    ref = oracle.attention_rows(Q, K, V, ref_mask, scale, items)
    O = o.reshape(B * H, S, d).float().cpu().numpy()
    errs = []
    for (bh, i), blk in ref.items():
        got = O[bh, i * 64: i * 64 + blk.shape[0]]
        assert np.isfinite(got).all()
        errs.append(np.abs(got - blk))
    e = np.concatenate([x.reshape(-1) for x in errs])
    assert e.max() <= max_abs, f"max abs err {e.max()}"
    assert e.mean() <= mean_abs, f"mean abs err {e.mean()}"
    return o, float(e.max()), float(e.mean())


def small_inputs(name, dtype=None, **kw):
    w = get_workload(name, **kw)
    if dtype is not None:
        w = w.replace(dtype=dtype)
    x = make_inputs(w)
    return w, x["q"].cuda(), x["k"].cuda(), x["v"].cuda()


# ------------------------------------------------------------------ pooling

@pytest.mark.parametrize("dtype,d,S", [("bf16", 128, 1000), ("bf16", 64, 64), ("f32", 64, 1024), ("f32", 128, 130)])
def test_block_means_parity(dtype, d, S):
    w, q, k, v = small_inputs("single", dtype=dtype, H=3, S=S, d=d, frame_len=max(S // 2, 1), region_len=64)
    got = fv.block_means(q).reshape(3, -1, d).cpu().numpy()
    ref = oracle.pool_blocks(q.reshape(3, S, d), 64)
    # The kernel adds four rows per thread in fp32 (bf16 input; fp64 for fp32 input) and the
    # partial sums in fp64: each partial is off by at most 3 ulp-halves of its magnitude, so
    # |err| <= 3 * 2^-24 * mean(|x|) per column (plus fp64 rounding).
    bound = 3 * 2.0 ** -24 * oracle.pool_blocks(q.abs().reshape(3, S, d), 64) + 1e-14
    if dtype == "f32":
        bound = 1e-14 * (1 + np.abs(ref))
    assert np.all(np.abs(got - ref) <= bound), float((np.abs(got - ref) / bound).max())


# ------------------------------------------------------------------ router

ROUTE_CASES = [
    ("tiny", {}, fv.RouteConfig(p=0.9)),
    ("tiny", {"alpha": ("const", 0.3)}, fv.RouteConfig(p=0.9)),
    ("single", {"H": 4, "S": 2000}, fv.RouteConfig(p=0.9)),
    ("single", {"H": 3, "S": 4096, "seed": 7}, fv.RouteConfig(p=0.5, force_diag=False)),
    ("single", {"H": 2, "S": 3000}, fv.RouteConfig(p=0.95, local_window=2)),
    ("single", {"H": 2, "S": 1560 * 2, "frame_len": 1560}, fv.RouteConfig(p=0.8, frame_len=1560, frame_window=0,
                                                                            force_first_frame=True)),
    ("single", {"H": 2, "S": 1000}, fv.RouteConfig(p=1.0)),
    ("single", {"H": 1, "S": 40}, fv.RouteConfig(p=0.9)),            # a single, partial block
    ("single", {"B": 2, "H": 2, "S": 64 * 9}, fv.RouteConfig(p=0.7)),  # odd block count: half tile
]


@pytest.mark.parametrize("name,kw,cfg", ROUTE_CASES)
def test_route_parity(name, kw, cfg):
    w, q, k, _ = small_inputs(name, **kw)
    check_route(q, k, cfg)


@pytest.mark.parametrize("fl,topk,fw,first", [(900, 2, 1, True), (1560, 1, 0, False), (640, 3, -1, True)])
def test_frame_mode_parity(fl, topk, fw, first):
    S = fl * 5 - 37
    w, q, k, _ = small_inputs("long", H=2, S=S, frame_len=fl, region_len=256)
    cfg = fv.RouteConfig(mode="frame_topk", topk_frames=topk, frame_len=fl, frame_window=fw,
                         force_first_frame=first, force_diag=True)
    check_route(q, k, cfg)


TOPK_CASES = [
    ("single", {"H": 3, "S": 3000}, fv.RouteConfig(mode="topk", topk_blocks=8, local_window=2, force_diag=False)),
    ("single", {"H": 2, "S": 8192, "alpha": ("const", 0.3)}, fv.RouteConfig(mode="topk", topk_blocks=5)),
    ("tiny", {}, fv.RouteConfig(mode="topk", topk_blocks=16, force_diag=False)),        # k = nb: dense
    ("single", {"H": 2, "S": 700}, fv.RouteConfig(mode="topk", topk_blocks=1, force_diag=False)),
]


@pytest.mark.parametrize("name,kw,cfg", TOPK_CASES)
def test_topk_blocks_parity(name, kw, cfg):
    w, q, k, v = small_inputs(name, **kw)
    csr, gm, r = check_route(q, k, cfg)
    if cfg.topk_blocks >= w.nb:
        assert gm.all()
    if w.dtype == "bf16":
        check_attention(q, k, v, csr, r, gm, 1.0 / np.sqrt(w.d))


# Slack-aware augmentation of 128-row tiles: the GPU's base routing is checked as above; the
# augmented sets must equal the oracle's (augmentation of the oracle's base) on every row whose
# tile has no near-tie, and on every row be a valid augmentation of the GPU's own base sets.
SASA_CASES = [
    ("single", {"H": 3, "S": 3000}, fv.RouteConfig(p=0.8, sasa_coef=0.5, sasa_trigger=1)),
    ("single", {"H": 2, "S": 8192}, fv.RouteConfig(p=0.9, sasa_coef=1.0, sasa_trigger=1)),
    ("dit", {"H": 3, "S": 1560 * 2}, fv.RouteConfig(p=0.9, sasa_coef=0.75, sasa_trigger=2)),
    ("single", {"H": 3, "S": 64 * 7 + 5, "d": 64}, fv.RouteConfig(p=0.7, sasa_coef=0.3, sasa_trigger=1)),
    ("single", {"H": 3, "S": 3000}, fv.RouteConfig(mode="topk", topk_blocks=6, sasa_coef=0.5, sasa_trigger=0)),
    ("single", {"H": 2, "S": 2048}, fv.RouteConfig(p=0.9, sasa_coef=0.5, sasa_trigger=1000)),
    ("single", {"H": 2, "S": 64 * 40, "alpha": ("const", 0.3)}, fv.RouteConfig(p=0.6, sasa_coef=0.7)),
]


@pytest.mark.parametrize("name,kw,cfg", SASA_CASES)
def test_sasa_parity(name, kw, cfg):
    w, q, k, v = small_inputs(name, **kw)
    B, H, S, d = q.shape
    _, gb, _ = check_route(q, k, dataclasses.replace(cfg, sasa_coef=0.0))
    csr = fv.route(q, k, cfg)
    assert fv.read_status(csr) == 0
    gm = gpu_mask(csr)
    oc = to_oracle_cfg(cfg)
    r = oracle.route(q.reshape(B * H, S, d), k.reshape(B * H, S, d), oc)
    key = r["pi"] if cfg.mode == "topp" else r["scores"]
    nb = w.nb
    for bh in range(B * H):
        for i in range(nb):
            if i ^ 1 >= nb:
                assert np.array_equal(gm[bh, i], gb[bh, i])
            else:
                assert oracle.valid_sasa_row(key[bh, i], gb[bh, i], gb[bh, i ^ 1], gm[bh, i], cfg.sasa_coef,
                                             cfg.sasa_trigger, cfg.mode), (bh, i)
    diff = np.any(gm != r["mask"], axis=2)
    bad = diff & ~r["near_tie"]
    assert not bad.any(), f"{int(bad.sum())} non-tie rows differ, e.g. {np.argwhere(bad)[:5].tolist()}"
    if cfg.sasa_trigger > nb:
        assert np.array_equal(gm, gb)
    # the tile costs (unions) do not change; the bookkeeping follows the augmented sets
    base = fv.route(q, k, dataclasses.replace(cfg, sasa_coef=0.0))
    np.testing.assert_array_equal(csr.tile_cost.cpu().numpy(), base.tile_cost.cpu().numpy())
    check_bookkeeping_properties(csr, gm)
    if not diff.any():
        rp, ci = oracle.csr_from_mask(r["mask"])
        np.testing.assert_array_equal(csr.row_ptr.cpu().numpy(), rp)
        np.testing.assert_array_equal(csr.col_idx[: len(ci)].cpu().numpy(), ci)
        np.testing.assert_array_equal(csr.head_load.cpu().numpy(), oracle.head_loads(r["mask"]))
        costs = oracle.tile_costs(r["mask"])
        np.testing.assert_array_equal(csr.tile_order.cpu().numpy(), oracle.lpt_order(costs))
    check_attention(q, k, v, csr, r, gm, 1.0 / np.sqrt(d))


# Token-exact frame mode: the same CSR as the block-granular frame mode, per-entry codes equal to
# the oracle's, and attention against the oracle's dense token mask.
EXACT_CASES = [
    ("single", {"H": 2, "S": 3000, "frame_len": 900}, dict(topk_frames=2, frame_window=-1, force_first_frame=False)),
    ("dit", {"H": 2, "S": 1560 * 2}, dict(topk_frames=1, frame_window=0, force_first_frame=True)),
    ("single", {"H": 3, "S": 64 * 20 + 9, "d": 64, "frame_len": 200}, dict(topk_frames=1, frame_window=-1,
                                                                         force_first_frame=False, local_window=1)),
    ("tiny", {"frame_len": 200}, dict(topk_frames=2, frame_window=-1, force_first_frame=True)),   # fp32 path
]


@pytest.mark.parametrize("name,kw,extra", EXACT_CASES)
def test_frame_exact_parity(name, kw, extra):
    w, q, k, v = small_inputs(name, **kw)
    B, H, S, d = q.shape
    force_diag = extra.pop("force_diag", True)
    cfg = fv.RouteConfig(mode="frame_topk", frame_len=w.frame_len, frame_exact=True, force_diag=force_diag, **extra)
    csr, gm, r = check_route(q, k, cfg, csr=fv.alloc_csr(B, H, S, q.device, codes=True))
    assert not r["near_tie"].any()                      # these cases have no near-tie frames
    oc = to_oracle_cfg(cfg)
    bf = oracle.block_forced(S, oc)
    rp, ci = oracle.csr_from_mask(r["mask"])
    want = np.array([oracle.frame_entry_code(r["frame_sets"][row // (w.nb)], bf, row % w.nb, int(ci[e]), S, oc)
                     for row in range(B * H * w.nb) for e in range(rp[row], rp[row + 1])], dtype=np.int64)
    np.testing.assert_array_equal(csr.col_code[: len(ci)].cpu().numpy().astype(np.int64), want)
    o = fv.sparse_attn(q, k, v, csr)
    assert fv.read_status(csr) == 0
    Q, K, V = (t.reshape(B * H, S, d).cpu() for t in (q, k, v))
    tok = np.stack([oracle.frame_token_mask(r["frame_sets"][bh], S, oc) for bh in range(B * H)])
    ref = oracle.attention_dense_mask(Q, K, V, tok, 1.0 / np.sqrt(d))
    e = np.abs(o.reshape(B * H, S, d).float().cpu().numpy() - ref)
    lim = (MAX_ABS_F32, MAX_ABS_F32) if w.dtype == "f32" else (MAX_ABS_BF16, MEAN_ABS_BF16)
    assert e.max() <= lim[0] and e.mean() <= lim[1], (e.max(), e.mean())
    # the block-granular answer differs where a kept block straddles a frame that is not kept
    blk = np.stack([np.repeat(np.repeat(r["mask"][bh], 64, 0), 64, 1)[:S, :S] for bh in range(B * H)])
    assert (blk & ~tok).any()


def test_route_deterministic():
    w, q, k, _ = small_inputs("single", H=3, S=4000, alpha=("const", 0.2))
    a = fv.route(q, k, fv.RouteConfig(p=0.9))
    b = fv.route(q, k, fv.RouteConfig(p=0.9))
    torch.cuda.synchronize()
    for f in ("row_ptr", "head_load", "tile_cost", "tile_order", "nnz"):
        assert torch.equal(getattr(a, f), getattr(b, f)), f
    n = int(a.nnz.item())
    assert torch.equal(a.col_idx[:n], b.col_idx[:n])


# ------------------------------------------------------------------ attention

ATTN_CASES = [
    ("single", {"H": 2, "S": 1000}, fv.RouteConfig(p=0.9)),
    ("single", {"H": 2, "S": 2048, "alpha": ("const", 0.5)}, fv.RouteConfig(p=0.9)),
    ("single", {"H": 3, "S": 64 * 7 + 5, "d": 64}, fv.RouteConfig(p=0.8, local_window=1)),
    ("single", {"H": 1, "S": 40}, fv.RouteConfig(p=0.9)),
    ("dit", {"H": 3, "S": 1560 * 2}, fv.RouteConfig(p=0.9)),
    ("single", {"B": 2, "H": 2, "S": 64 * 9 + 30}, fv.RouteConfig(p=0.8)),        # B > 1, odd block count
]


@pytest.mark.parametrize("name,kw,cfg", ATTN_CASES)
def test_attention_parity_bf16(name, kw, cfg):
    w, q, k, v = small_inputs(name, **kw)
    csr, gm, r = check_route(q, k, cfg)
    check_attention(q, k, v, csr, r, gm, 1.0 / np.sqrt(w.d))


def test_attention_p1_equals_dense_bf16():
    w, q, k, v = small_inputs("single", H=2, S=1100)
    csr, gm, r = check_route(q, k, fv.RouteConfig(p=1.0))
    assert gm.all()
    o = fv.sparse_attn(q, k, v, csr)
    dense = torch.nn.functional.scaled_dot_product_attention(q.double(), k.double(), v.double())
    e = (o.double() - dense).abs()
    assert e.max().item() <= MAX_ABS_BF16 and e.mean().item() <= MEAN_ABS_BF16


@pytest.mark.parametrize("p", [0.9, 1.0])
def test_tiny_fp32_path(p):
    w, q, k, v = small_inputs("tiny", alpha=("const", 0.4))
    csr, gm, r = check_route(q, k, fv.RouteConfig(p=p))
    check_attention(q, k, v, csr, r, gm, 1.0 / 8.0, max_abs=MAX_ABS_F32, mean_abs=MAX_ABS_F32)


def test_attention_lse_and_determinism():
    w, q, k, v = small_inputs("single", H=2, S=1500, alpha=("const", 0.7))
    csr = fv.route(q, k, fv.RouteConfig(p=0.9))
    lse = torch.empty((1, 2, 1500), dtype=torch.float32, device="cuda")
    o1 = fv.sparse_attn(q, k, v, csr, lse=lse)
    o2 = fv.sparse_attn(q, k, v, csr)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    gm = gpu_mask(csr)
    # lse of query block 3 of head 1, rebuilt from the selected keys
    Q, K = q[0, 1].double().cpu(), k[0, 1].double().cpu()
    cols = np.concatenate([np.arange(j * 64, min(1500, j * 64 + 64)) for j in np.nonzero(gm[1, 3])[0]])
    s = (Q[192:256] @ K[cols].T) / np.sqrt(128)
    ref = torch.logsumexp(s, dim=1).numpy()
    np.testing.assert_allclose(lse[0, 1, 192:256].cpu().numpy(), ref, atol=2e-2)


# ------------------------------------------------------------------ full size

@pytest.mark.slow
def test_full_size_dit_layer_sampled():
    """The benchmarked layer (B=1, H=40, S=32760, d=128, bf16, p=0.9): every block list
    against the oracle, attention on a seeded sample of query blocks."""
    w = get_workload("dit")
    x = make_inputs(w, device="cuda")
    q, k, v = x["q"], x["k"], x["v"]
    csr, gm, r = check_route(q, k, fv.RouteConfig(p=0.9))
    rng = np.random.default_rng(0)
    items = [(int(bh), int(i)) for bh, i in zip(rng.integers(0, 40, 48), rng.integers(0, w.nb, 48))]
    items += [(0, w.nb - 1), (39, w.nb - 1)]                      # the ragged last block
    _, emax, emean = check_attention(q, k, v, csr, r, gm, 1.0 / np.sqrt(128), items=items)


@pytest.mark.slow
def test_full_length_long_frame_mode_sampled_heads():
    """S=75600 (21 frames x 3600 tokens), frame top-k=4 with frames +-1 and frame 0, on 4 of
    the 40 heads (same per-head generator)."""
    w = get_workload("long", H=4)
    x = make_inputs(w, device="cuda")
    q, k, v = x["q"], x["k"], x["v"]
    cfg = fv.RouteConfig(mode="frame_topk", topk_frames=4, frame_len=3600, frame_window=1, force_first_frame=True)
    csr, gm, r = check_route(q, k, cfg)
    rng = np.random.default_rng(1)
    items = [(int(bh), int(i)) for bh, i in zip(rng.integers(0, 4, 12), rng.integers(0, w.nb, 12))]
    check_attention(q, k, v, csr, r, gm, 1.0 / np.sqrt(128), items=items)


# The three register/shared-memory variants of the per-row cut: rows of <= 512 blocks, of
# 513..1280 blocks (the long layer's 1182) and of more than 1280 blocks (shared-memory cut, also
# past 2048 blocks, where a row's bitmask has more than 64 words), each with the full block
# lists checked and attention on a sample of query blocks.
@pytest.mark.slow
@pytest.mark.parametrize("S,extra", [
    (75600, {}),                                                        # nb = 1182
    (1290 * 64 + 17, {}),                                               # nb = 1291: shared-memory cut
    (2100 * 64, {}),                                                    # nb = 2100: 66 mask words per row
    (700 * 64, {"mode": "topk", "topk_blocks": 40}),                    # nb = 700, top-k
    (700 * 64 + 5, {"sasa_coef": 0.5, "sasa_trigger": 2}),               # nb = 701, tile augmentation
])
def test_long_rows_parity(S, extra):
    w = get_workload("long", H=1, S=S, d=64)
    x = make_inputs(w, device="cuda")
    q, k, v = x["q"], x["k"], x["v"]
    cfg = fv.RouteConfig(p=0.9, **extra)
    if cfg.sasa_coef > 0:
        B, H, S_, d = q.shape
        _, gb, _ = check_route(q, k, dataclasses.replace(cfg, sasa_coef=0.0))
        csr = fv.route(q, k, cfg)
        assert fv.read_status(csr) == 0
        gm = gpu_mask(csr)
        r = oracle.route(q.reshape(B * H, S_, d), k.reshape(B * H, S_, d), to_oracle_cfg(cfg))
        for i in range(w.nb):
            if i ^ 1 < w.nb:
                assert oracle.valid_sasa_row(r["pi"][0, i], gb[0, i], gb[0, i ^ 1], gm[0, i], cfg.sasa_coef,
                                             cfg.sasa_trigger, "topp"), i
        assert not (np.any(gm != r["mask"], axis=2) & ~r["near_tie"]).any()
    else:
        csr, gm, r = check_route(q, k, cfg)
    rng = np.random.default_rng(2)
    items = [(0, int(i)) for i in rng.integers(0, w.nb, 10)] + [(0, w.nb - 1)]
    check_attention(q, k, v, csr, r, gm, 1.0 / np.sqrt(64), items=items)
