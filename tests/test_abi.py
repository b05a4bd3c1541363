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


def test_header_is_plain_c(tmp_path):
    # the boundary has no C++ or torch types: the header compiles as C99 with warnings as errors
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use.c"
    src.write_text('#include "fvattn.h"\nint main(void) { return fvattn_version() > 0 ? 0 : 1; }\n')
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.dirname(HEADER),
                        "-c", str(src), "-o", str(tmp_path / "use.o")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_checked_build_exports_every_declared_symbol():
    # libfvattn_debug.so (-DFVATTN_DEBUG) is a drop-in for the same boundary
    import ctypes
    assert os.path.exists(_lib.DEBUG_LIB_PATH), "build it with `python -m block_sparse_top_fvattn_b200.build --debug`"
    dbg = ctypes.CDLL(_lib.DEBUG_LIB_PATH)
    for n in declared_functions():
        assert hasattr(dbg, n), n


def test_version_and_status_strings(lib):
    assert lib.fvattn_version() >> 16 == 1
    for code in range(0, -6, -1):
        s = _lib.status_string(code)
        assert s and s != "unknown status"
    assert _lib.status_string(12345) == "unknown status"


def test_block_scores_sizes_and_host_checks(lib):
    s = shape(B=1, H=2, S=1000)                 # nb = 16, ld = 32
    assert lib.fvattn_block_scores_ld(ctypes.byref(s)) == 32
    ws = lib.fvattn_block_scores_workspace_bytes(ctypes.byref(s))
    assert ws >= 2 * (2 * 5 * 16 * 128) + 2 * (2 * 16 * 4)     # Q and K slices, exponents
    bad = shape(d=96)
    assert lib.fvattn_block_scores_ld(ctypes.byref(bad)) == 0
    assert lib.fvattn_block_scores_workspace_bytes(ctypes.byref(bad)) == 0
    buf = ctypes.create_string_buffer(4096)
    p = ctypes.cast(buf, ctypes.c_void_p)
    st = lib.fvattn_block_scores(None, p, ctypes.byref(s), p, p, ws, p, None)
    assert st == _lib.FVATTN_ERR_INVALID
    st = lib.fvattn_block_scores(p, p, ctypes.byref(bad), p, p, ws, p, None)
    assert st == _lib.FVATTN_ERR_UNSUPPORTED


def test_timeout_checks_reject_bad_arguments_on_the_host(lib):
    s = shape(B=1, H=2, S=1000)
    buf = ctypes.create_string_buffer(4096)
    p = ctypes.cast(ctypes.addressof(buf) + (-ctypes.addressof(buf)) % 256, ctypes.c_void_p)
    csr = _fake_csr(16 * 16 * 2)
    assert lib.fvattn_sparse_attn_timeout_check(p, p, p, ctypes.byref(s), ctypes.byref(csr), p, 0, None) == \
        _lib.FVATTN_ERR_INVALID
    f32 = shape(dtype=1)
    assert lib.fvattn_sparse_attn_timeout_check(p, p, p, ctypes.byref(f32), ctypes.byref(csr), p, 4, None) == \
        _lib.FVATTN_ERR_UNSUPPORTED
    assert lib.fvattn_sparse_attn_timeout_check(p, p, p, ctypes.byref(shape(d=96)), ctypes.byref(csr), p, 4,
                                                None) == _lib.FVATTN_ERR_UNSUPPORTED
    ws = lib.fvattn_block_scores_workspace_bytes(ctypes.byref(s))
    assert lib.fvattn_block_scores_timeout_check(p, p, ctypes.byref(s), p, p, ws, p, 0, None) == \
        _lib.FVATTN_ERR_INVALID
    assert lib.fvattn_block_scores_timeout_check(None, p, ctypes.byref(s), p, p, ws, p, 4, None) == \
        _lib.FVATTN_ERR_INVALID
    assert lib.fvattn_block_scores_timeout_check(p, p, ctypes.byref(s), p, p, ws - 1, p, 4, None) == \
        _lib.FVATTN_ERR_CAPACITY


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
    # Q and K score slices (5 int8 planes of 128-byte rows), fp64 logits (rows of 32), bitmasks
    slices = 2 * 5 * 16 * 128
    assert ws >= 2 * slices + 2 * 16 * 32 * 8 + 2 * 16 * 1 * 4 + 2 * 16 * 4
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
    dict(frame_exact=1),                                          # token-exact needs frame mode
    dict(mode=1, frame_len=256, topk_frames=2, frame_exact=2),
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
    exact = cfg(mode=1, frame_len=256, topk_frames=2, frame_exact=1)       # col_code is NULL in csr
    ws_e = lib.fvattn_route_workspace_bytes(ctypes.byref(s), ctypes.byref(exact))
    assert ws_e > 0
    assert lib.fvattn_route(P, P, ctypes.byref(s), ctypes.byref(exact), ctypes.byref(csr), P, ws_e, None) == -1
    assert lib.fvattn_route(P, P, ctypes.byref(shape(block=32)), ctypes.byref(c), ctypes.byref(csr), P, ws,
                            None) == -2


def test_two_stage_route_rejects_on_host_before_any_launch(lib):
    s, c = shape(), cfg()                       # S = 1000: nb = 16
    ws = lib.fvattn_route_workspace_bytes(ctypes.byref(s), ctypes.byref(c))
    csr = _fake_csr(lib.fvattn_csr_max_nnz(ctypes.byref(s)))
    P = 4096
    pool = lib.fvattn_route_pool
    assert pool(None, P, ctypes.byref(s), ctypes.byref(c), 0, 16, P, ws, None) == -1
    assert pool(P, P, ctypes.byref(s), ctypes.byref(c), 0, 16, P, ws - 1, None) == -3
    for b0, b1 in ((-1, 4), (4, 4), (10, 17), (5, 3)):
        assert pool(P, P, ctypes.byref(s), ctypes.byref(c), b0, b1, P, ws, None) == -1
    assert pool(P, P, ctypes.byref(shape(d=96)), ctypes.byref(c), 0, 16, P, ws, None) == -2
    fin = lib.fvattn_route_finish
    assert fin(ctypes.byref(s), ctypes.byref(c), None, P, ws, None) == -1
    assert fin(ctypes.byref(s), ctypes.byref(c), ctypes.byref(csr), None, ws, None) == -1
    assert fin(ctypes.byref(s), ctypes.byref(c), ctypes.byref(_fake_csr(10)), P, ws, None) == -3


def test_attention_and_status_reject_on_host(lib):
    s = shape()
    csr = _fake_csr(1)
    P = 4096
    assert lib.fvattn_sparse_attn(P, P, None, ctypes.byref(s), ctypes.byref(csr), P, None, None) == -1
    assert lib.fvattn_sparse_attn(P, P, P + 8, ctypes.byref(s), ctypes.byref(csr), P, None, None) == -1
    assert lib.fvattn_sparse_attn(P, P, P, ctypes.byref(shape(d=80)), ctypes.byref(csr), P, None, None) == -2
    assert lib.fvattn_block_means(None, ctypes.byref(s), P, None) == -1
    assert lib.fvattn_read_status(None, None) == -1


# ---------------------------------------------------------------- runtime load balancing plan (host)

@pytest.mark.parametrize("seed", range(25))
def test_rlb_plan_matches_oracle(lib, seed):
    import numpy as np
    import oracle
    import block_sparse_top_fvattn_b200 as fv
    rng = np.random.default_rng(seed)
    R, Hl = int(rng.integers(1, 9)), int(rng.integers(1, 9))
    loads = rng.integers(0, 5000, size=(R, Hl)) * (rng.random((R, Hl)) < 0.85)
    if seed % 5 == 0:
        loads[:, :] = rng.integers(0, 3, size=(R, Hl))       # many ties
    target = float(rng.choice([1.0, 1.02, 1.1, 1.3]))
    budget = int(rng.integers(0, 4))
    got = fv.rlb_plan(loads, target, budget)
    want = oracle.rlb_plan(loads, target, budget)
    assert got[0] == [tuple(m) for m in want[0]]
    assert got[1] == want[1]


def test_rlb_plan_rejects_bad_arguments(lib):
    import numpy as np
    loads = np.array([[5, 1], [1, 1]], dtype=np.int64)
    moves = np.zeros(3 * 4, dtype=np.int32)
    n = ctypes.c_int32(-7)

    def call(ld=loads, R=2, Hl=2, target=1.05, budget=1, mv=moves, cap=4):
        return lib.fvattn_rlb_plan(ld.ctypes.data if ld is not None else None, R, Hl, target, budget,
                                   mv.ctypes.data if mv is not None else None, cap, ctypes.byref(n), None)

    assert call() == 0 and n.value == 1
    assert call(ld=None) == -1
    assert call(R=0) == -1 and call(Hl=0) == -1
    assert call(target=0.99) == -1 and call(target=float("nan")) == -1 and call(target=float("inf")) == -1
    assert call(budget=-1) == -1
    assert call(ld=np.array([[5, -1], [1, 1]], dtype=np.int64)) == -1
    assert call(cap=1) == -3                              # needs ranks * min(budget, heads) = 2 entries
    assert call(budget=0, cap=0, mv=None) == 0 and n.value == 0


def test_lazy_router_refresh_schedule():
    # which diffusion steps recompute the routing (no GPU needed: the schedule only)
    import block_sparse_top_fvattn_b200 as fv

    class FakeCsr:
        B, H, S = 1, 2, 1000

    lr = fv.LazyRouter(fv.RouteConfig(), refresh_every=4)
    assert lr.should_refresh(0, (1, 2, 1000))                  # nothing routed yet
    lr.csr, lr.last_refresh = FakeCsr(), 0
    assert [s for s in range(1, 10) if lr.should_refresh(s, (1, 2, 1000))] == [4, 5, 6, 7, 8, 9]
    lr.last_refresh = 4
    assert [s for s in range(5, 13) if lr.should_refresh(s, (1, 2, 1000))] == [8, 9, 10, 11, 12]
    assert lr.should_refresh(5, (1, 2, 2000))                  # a new shape always routes
    assert lr.should_refresh(3, (1, 2, 1000))                  # a step before the last refresh
    with pytest.raises(ValueError):
        fv.LazyRouter(refresh_every=0)
