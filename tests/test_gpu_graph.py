"""The router and the attention captured once in a CUDA graph and replayed.

Every call of the library is stream-ordered (kernel launches and memsets on the caller's
stream, no host synchronisation), so one step, route and attention, can be captured into a
CUDA graph with static input and output buffers and replayed after new inputs are copied in.
The replayed CSR and output are checked against the oracle on each new input draw, as the direct
calls are."""
import numpy as np
import pytest
import torch

import block_sparse_top_fvattn_b200 as fv
from workloads import make_inputs
from test_gpu_parity import compare_attention, compare_csr, small_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fv.load()


@pytest.mark.parametrize("cfg", [fv.RouteConfig(p=0.9), fv.RouteConfig(mode="topk", topk_blocks=6)])
def test_route_and_attention_replayed_from_a_cuda_graph(cfg):
    w, q, k, v = small_inputs("single", H=3, S=2500)
    csr = fv.alloc_csr(1, w.H, w.S, "cuda")
    ws = torch.empty(fv.workspace_bytes(q, cfg), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    fv.route(q, k, cfg, csr=csr, workspace=ws)            # first calls outside the capture
    fv.sparse_attn(q, k, v, csr, out=out)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fv.route(q, k, cfg, csr=csr, workspace=ws)
        fv.sparse_attn(q, k, v, csr, out=out)
    for seed in (11, 12):
        x = make_inputs(w.replace(seed=seed))
        q.copy_(x["q"]), k.copy_(x["k"]), v.copy_(x["v"])
        g.replay()
        torch.cuda.synchronize()
        assert fv.read_status(csr) == 0
        csr_r, gm, r = compare_csr(csr, q, k, cfg)
        compare_attention(out, q, k, v, r, gm, 1.0 / np.sqrt(w.d))
    del g
