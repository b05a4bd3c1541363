"""The C ABI library on a machine without a GPU: it loads, exports every entry point that
include/fvattn.h declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

from block_sparse_top_fvattn_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fvattn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fvattn_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("fvattn_route", "fvattn_sparse_attn", "fvattn_read_status", "fvattn_status_string",
              "fvattn_csr_max_nnz", "fvattn_route_workspace_bytes"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_version_and_status_strings(lib):
    assert lib.fvattn_version() >> 16 == 1
    for code in range(0, -6, -1):
        s = _lib.status_string(code)
        assert s and s != "unknown status"
    assert _lib.status_string(12345) == "unknown status"


def shape(B=1, H=2, S=1000, d=128, block=64, dtype=0, scale=0.0):
    return _lib.Shape(B, H, S, d, block, dtype, scale)


def cfg(**kw):
    base = dict(mode=0, p=0.9, force_diag=1, local_window=0, frame_len=0, topk_frames=0, frame_window=-1,
                force_first_frame=0)
    base.update(kw)
    return _lib.RouteCfg(**base)


def test_sizes_on_host(lib):
    s = shape(B=2, H=3, S=1000)          # nb = 16
    assert lib.fvattn_csr_max_nnz(ctypes.byref(s)) == 6 * 16 * 16
    assert lib.fvattn_num_tiles(ctypes.byref(s)) == 6 * 8
    s = shape(S=65)                      # nb = 2 with a 1-token tail
    assert lib.fvattn_num_tiles(ctypes.byref(s)) == 2 * 1
    ws = lib.fvattn_route_workspace_bytes(ctypes.byref(shape(S=1000)), ctypes.byref(cfg()))
    means = 2 * 16 * 128 * 8
    assert ws >= 2 * means + 2 * 16 * 1 * 4 + 2 * 16 * 4
    wf = lib.fvattn_route_workspace_bytes(ctypes.byref(shape(S=1000)),
                                          ctypes.byref(cfg(mode=1, frame_len=250, topk_frames=2)))
    assert wf > ws


@pytest.mark.parametrize("bad,code", [
    (dict(block=32), _lib.FVATTN_ERR_UNSUPPORTED),
    (dict(d=96), _lib.FVATTN_ERR_UNSUPPORTED),
    (dict(S=0), _lib.FVATTN_ERR_INVALID),
    (dict(H=-1), _lib.FVATTN_ERR_INVALID),
    (dict(dtype=7), _lib.FVATTN_ERR_INVALID),
    (dict(scale=float("nan")), _lib.FVATTN_ERR_INVALID),
])
def test_invalid_shapes(lib, bad, code):
    s = shape(**bad)
    assert lib.fvattn_csr_max_nnz(ctypes.byref(s)) == code
    assert lib.fvattn_route_workspace_bytes(ctypes.byref(s), ctypes.byref(cfg())) == 0


@pytest.mark.parametrize("bad", [
    dict(p=0.0), dict(p=-0.5), dict(p=float("nan")), dict(local_window=-1), dict(mode=5),
    dict(frame_window=0),                                   # neighbour frames without a frame length
    dict(mode=1, frame_len=32, topk_frames=2),              # frames shorter than a block
    dict(mode=1, frame_len=256, topk_frames=0),
    dict(sasa_coef=-0.1), dict(sasa_coef=1.5), dict(sasa_coef=float("nan")), dict(sasa_trigger=-1),
    dict(mode=1, frame_len=256, topk_frames=2, sasa_coef=0.5),   # frame mode has no per-block order
])
def test_invalid_configs(lib, bad):
    assert lib.fvattn_route_workspace_bytes(ctypes.byref(shape()), ctypes.byref(cfg(**bad))) == 0


def test_sasa_limits(lib):
    # accepted in Top-p and top-k modes up to 1280 blocks per row, rejected (unsupported) above
    ok = cfg(sasa_coef=1.0, sasa_trigger=0)
    assert lib.fvattn_route_workspace_bytes(ctypes.byref(shape()), ctypes.byref(ok)) > 0
    assert lib.fvattn_route_workspace_bytes(ctypes.byref(shape()), ctypes.byref(cfg(mode=2, topk_blocks=3,
                                                                                   sasa_coef=0.5))) > 0
    assert lib.fvattn_route_workspace_bytes(ctypes.byref(shape(S=1280 * 64)), ctypes.byref(ok)) > 0
    assert lib.fvattn_route_workspace_bytes(ctypes.byref(shape(S=1280 * 64 + 1)), ctypes.byref(ok)) == 0
    assert lib.fvattn_route_workspace_bytes(ctypes.byref(shape(S=1280 * 64 + 1)), ctypes.byref(cfg())) > 0


def _fake_csr(cap):
    p = 4096                                                # aligned, never dereferenced on the host
    return _lib.Csr(p, p, cap, p, p, p, p, p)


def test_route_rejects_on_host_before_any_launch(lib):
    s, c = shape(), cfg()
    ws = lib.fvattn_route_workspace_bytes(ctypes.byref(s), ctypes.byref(c))
    csr = _fake_csr(lib.fvattn_csr_max_nnz(ctypes.byref(s)))
    P = 4096
    assert lib.fvattn_route(None, P, ctypes.byref(s), ctypes.byref(c), ctypes.byref(csr), P, ws, None) == -1
    assert lib.fvattn_route(P + 4, P, ctypes.byref(s), ctypes.byref(c), ctypes.byref(csr), P, ws, None) == -1
    assert lib.fvattn_route(P, P, ctypes.byref(s), ctypes.byref(c), ctypes.byref(csr), P, ws - 1, None) == -3
    small = _fake_csr(10)
    assert lib.fvattn_route(P, P, ctypes.byref(s), ctypes.byref(c), ctypes.byref(small), P, ws, None) == -3
    bad = cfg(p=0.0)
    assert lib.fvattn_route(P, P, ctypes.byref(s), ctypes.byref(bad), ctypes.byref(csr), P, ws, None) == -1
    assert lib.fvattn_route(P, P, ctypes.byref(shape(block=32)), ctypes.byref(c), ctypes.byref(csr), P, ws,
                            None) == -2


def test_attention_and_status_reject_on_host(lib):
    s = shape()
    csr = _fake_csr(1)
    P = 4096
    assert lib.fvattn_sparse_attn(P, P, None, ctypes.byref(s), ctypes.byref(csr), P, None, None) == -1
    assert lib.fvattn_sparse_attn(P, P, P + 8, ctypes.byref(s), ctypes.byref(csr), P, None, None) == -1
    assert lib.fvattn_sparse_attn(P, P, P, ctypes.byref(shape(d=80)), ctypes.byref(csr), P, None, None) == -2
    assert lib.fvattn_block_means(None, ctypes.byref(s), P, None) == -1
    assert lib.fvattn_read_status(None, None) == -1
