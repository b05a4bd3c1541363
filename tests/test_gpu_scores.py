"""fvattn_block_scores (the router's fp64 block scores from exact 8-bit integer slices on the
tensor cores) against the oracle's scaled dot products of the fp64 block means, element by
element, within a bound derived from the arithmetic: the pooling's fp32 partial sums of bf16
rows (error <= 3 * 2^-24 * mean|x| per mean) plus the slices' dropped terms (below 2^-30 *
2^(e_i + e_j), here bounded by 2^-24 * d * max|Qbar_i| * max|Kbar_j|). A wrong digit, level or
exponent moves a score by at least 2^-8 of its size. Also the stamped attention entry point
(per-CTA SM ids and busy intervals: same output as the plain call, valid stamps) and the
two-stage router (pooling by block ranges, then the rest: the same CSR as fvattn_route)."""
import importlib

import numpy as np
import pytest
import torch

import block_sparse_top_fvattn_b200 as fv
from test_gpu_parity import compare_csr
from workloads import get_workload, make_inputs

oroute = importlib.import_module("oracle.route")

pytestmark = pytest.mark.gpu

CASES = [
    ("tiny", {}),                                   # fp32, d = 64, S = 1024
    ("single", dict(H=2, S=3000)),                  # bf16, d = 128, ragged last block
    ("single", dict(H=2, S=2000, d=64)),            # bf16, d = 64 (slice rows half zero)
    ("dit", dict(H=2)),                             # bf16, S = 32760, peaked heads (large logits)
]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fv.load()


@pytest.mark.parametrize("name,over", CASES)
def test_block_scores_match_oracle(name, over):
    w = get_workload(name).replace(**over) if over else get_workload(name)
    d_ = make_inputs(w, device="cuda")
    q, k = d_["q"], d_["k"]
    B, H, S, d = q.shape
    got = fv.block_scores(q, k).cpu().numpy().reshape(B * H, -1, -(-S // 64))
    Q = q.reshape(B * H, S, d).cpu().double().numpy()
    K = k.reshape(B * H, S, d).cpu().double().numpy()
    scale = 1.0 / np.sqrt(d)
    qm, km = oroute.pool_blocks(Q, 64), oroute.pool_blocks(K, 64)
    want = oroute.block_scores(qm, km, scale)
    qa, ka = oroute.pool_blocks(np.abs(Q), 64), oroute.pool_blocks(np.abs(K), 64)
    pool_err = 3.0 * 2.0 ** -24 * (np.matmul(qa, np.abs(km).swapaxes(1, 2)) + np.matmul(np.abs(qm), ka.swapaxes(1, 2)))
    slice_err = 2.0 ** -24 * d * np.abs(qm).max(axis=2)[:, :, None] * np.abs(km).max(axis=2)[:, None, :]
    tol = scale * (1.01 * pool_err + slice_err) + 1e-300
    err = np.abs(got - want)
    worst = float((err / tol).max())
    assert worst <= 1.0, f"max |gpu - oracle| / bound = {worst:.3g} (max abs error {err.max():.3g})"
    # the bound is tight enough to mean something: far below the size of the scores
    assert float(tol.max()) < 1e-5 * max(1.0, float(np.abs(want).max()))


def test_block_scores_rejects_mismatched_inputs():
    q = torch.zeros(1, 1, 128, 64, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fv.block_scores(q, torch.zeros(1, 1, 128, 64, device="cuda", dtype=torch.float32))


def test_stamped_attention_equals_plain_and_stamps_are_valid():
    """fvattn_sparse_attn_stamped runs the same kernel: its output equals fvattn_sparse_attn's
    bit for bit, and every CTA reports an SM id below the device's SM count and start <= end."""
    w = get_workload("single").replace(H=4, S=4000)
    x = make_inputs(w, device="cuda")
    q, k, v = x["q"], x["k"], x["v"]
    csr = fv.route(q, k, fv.RouteConfig(p=0.9))
    o_plain = fv.sparse_attn(q, k, v, csr)
    o_st, stamps = fv.sparse_attn_stamped(q, k, v, csr)
    torch.cuda.synchronize()
    assert fv.read_status(csr) == 0
    assert torch.equal(o_plain, o_st)
    st = stamps.cpu().numpy()
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    assert st.shape[0] >= 1 and np.all(st[:, 0] >= 0) and np.all(st[:, 0] < nsm)
    assert np.all(st[:, 1] > 0) and np.all(st[:, 2] >= st[:, 1])
    imb = fv.sm_busy_imbalance(stamps)
    assert imb["imbalance"] >= 1.0 and imb["sms"] <= nsm


def test_stamped_attention_rejects_fp32():
    w = get_workload("tiny")
    x = make_inputs(w, device="cuda")
    csr = fv.route(x["q"], x["k"], fv.RouteConfig(p=0.9))
    with pytest.raises(fv.FvattnError):
        fv.sparse_attn_stamped(x["q"], x["k"], x["v"], csr)


SPLIT_CASES = [
    ("single", dict(H=3, S=3000), fv.RouteConfig(p=0.9), [(20, 47), (0, 20)]),                  # ragged tail last
    ("single", dict(H=2, S=4096), fv.RouteConfig(p=0.8, local_window=1), [(32, 64), (0, 8), (8, 32)]),
    ("single", dict(H=2, S=3120, frame_len=1560), fv.RouteConfig(mode="frame_topk", topk_frames=1, frame_len=1560,
                                                                   frame_window=0, force_first_frame=True),
     [(25, 49), (0, 25)]),
    # range ends inside frames (blocks 10 and 30 start at tokens 640 and 1920, inside frames 0
    # and 2 of 900 tokens) and a ragged last block (tokens 2944-2999)
    ("single", dict(H=2, S=3000, frame_len=900, region_len=128),
     fv.RouteConfig(mode="frame_topk", topk_frames=2, frame_len=900, frame_window=-1), [(30, 47), (0, 10), (10, 30)]),
    ("single", dict(H=2, S=3000, frame_len=900, region_len=128),
     fv.RouteConfig(mode="frame_topk", topk_frames=1, frame_len=900, frame_window=0, force_first_frame=True,
                    frame_exact=True), [(10, 30), (30, 47), (0, 10)]),
    ("single", dict(H=3, S=2500), fv.RouteConfig(mode="topk", topk_blocks=6), [(0, 13), (13, 40)]),
]


@pytest.mark.parametrize("name,over,cfg,ranges", SPLIT_CASES)
def test_split_route_equals_route(name, over, cfg, ranges):
    """fvattn_route_pool over block ranges in any order, then fvattn_route_finish: the CSR (and in
    token-exact frame mode the entry codes) against the oracle's router on the same inputs, and
    bit for bit equal to fvattn_route's (the same kernels on the same blocks)."""
    w = get_workload(name).replace(**over)
    x = make_inputs(w, device="cuda")
    q, k = x["q"], x["k"]
    a = fv.route(q, k, cfg)
    ws = torch.empty(fv.workspace_bytes(q, cfg), dtype=torch.uint8, device="cuda")
    for b0, b1 in ranges:
        fv.route_pool(q, k, cfg, b0, b1, ws)
    b = fv.route_finish(q, cfg, ws)
    torch.cuda.synchronize()
    assert fv.read_status(a) == 0 and fv.read_status(b) == 0
    compare_csr(b, q, k, cfg)
    for f in ("row_ptr", "head_load", "tile_cost", "tile_order", "nnz"):
        assert torch.equal(getattr(a, f), getattr(b, f)), f
    n = int(a.nnz.item())
    assert torch.equal(a.col_idx[:n], b.col_idx[:n])
    if cfg.frame_exact:
        assert torch.equal(a.col_code[:n], b.col_code[:n])


def test_route_pool_rejects_bad_ranges():
    w = get_workload("single").replace(H=1, S=1000)
    x = make_inputs(w, device="cuda")
    cfg = fv.RouteConfig(p=0.9)
    ws = torch.empty(fv.workspace_bytes(x["q"], cfg), dtype=torch.uint8, device="cuda")
    for b0, b1 in ((-1, 4), (4, 4), (10, 17), (5, 3)):
        with pytest.raises(fv.FvattnError):
            fv.route_pool(x["q"], x["k"], cfg, b0, b1, ws)
