"""fvattn_route_static_scratch: the router for callers that cannot allocate device memory
(a host that owns every byte of device memory in its own pool, or a plugin interface that
passes only input and output pointers). It must give exactly what fvattn_route gives, call
after call, although all calls share one static scratch array that keeps the previous
call's contents. Collected last so that a failure here stops nothing else."""
import ctypes

import pytest
import torch

import block_sparse_top_fvattn_b200 as fv
from block_sparse_top_fvattn_b200 import _lib
from workloads import get_workload, make_inputs

pytestmark = pytest.mark.gpu

FIELDS = ("row_ptr", "head_load", "tile_cost", "tile_order", "nnz")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _inputs(seed, **kw):
    w = get_workload("single", **kw)
    x = make_inputs(w, seed=seed)
    return x["q"].cuda(), x["k"].cuda()


def _static_route(q, k, cfg):
    lib = _lib.load()
    B, H, S, _ = q.shape
    csr = fv.alloc_csr(B, H, S, q.device)
    shp = fv.shape_of(q)
    c_cfg = cfg.to_c()
    c_csr = csr.to_c()
    st = lib.fvattn_route_static_scratch(q.data_ptr(), k.data_ptr(), ctypes.byref(shp), ctypes.byref(c_cfg),
                                         ctypes.byref(c_csr),
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, csr


def _same(a, b):
    torch.cuda.synchronize()
    for f in FIELDS:
        assert torch.equal(getattr(a, f), getattr(b, f)), f
    n = int(a.nnz.item())
    assert torch.equal(a.col_idx[:n], b.col_idx[:n])


def test_static_scratch_matches_route_on_two_calls_in_a_row():
    cfg = fv.RouteConfig(p=0.9, local_window=1)
    # two different problems back to back: the second call must not see the first's leftovers
    for seed, kw in ((11, dict(H=3, S=3000)), (12, dict(H=12, S=8192))):
        q, k = _inputs(seed, **kw)
        st, got = _static_route(q, k, cfg)
        assert st == 0, _lib.status_string(st)
        assert fv.read_status(got) == 0
        ref = fv.route(q, k, cfg)
        _same(got, ref)


def test_static_scratch_other_modes_on_a_dirty_array():
    # Frame top-k and fixed top-k use other parts of the scratch than Top-p (segment sums, frame
    # means, kept-frame bits); after a Top-p call has left its contents there, each must still
    # give exactly what fvattn_route gives.
    q, k = _inputs(14, H=4, S=3000, frame_len=900, region_len=128)
    cfgs = (fv.RouteConfig(p=0.8),
            fv.RouteConfig(mode="frame_topk", topk_frames=2, frame_len=900, frame_window=0, force_first_frame=True),
            fv.RouteConfig(mode="topk", topk_blocks=5, local_window=1),
            fv.RouteConfig(mode="frame_topk", topk_frames=1, frame_len=900, frame_window=-1))
    for cfg in cfgs:
        st, got = _static_route(q, k, cfg)
        assert st == 0, _lib.status_string(st)
        assert fv.read_status(got) == 0
        _same(got, fv.route(q, k, cfg))


def test_static_scratch_rejects_sizes_beyond_its_array():
    q, k = _inputs(13, H=40, S=8192)          # needs about 10 MiB of router scratch
    st, _ = _static_route(q, k, fv.RouteConfig(p=0.9))
    assert st == _lib.FVATTN_ERR_CAPACITY
