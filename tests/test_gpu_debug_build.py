"""The checked build (libfvattn_debug.so, compiled with -DFVATTN_DEBUG) on a B200.

Its attention kernels check the CSR lists of every tile before any role reads them: row offsets
non-decreasing and within the column array, key blocks in [0, nb), each list strictly
ascending. A failed check is written to the device status word as FVATTN_ERR_INVALID with the
check in status[1] (101 / 102 / 103), the tile is skipped, and nothing outside the arrays is
read, so a corrupted CSR becomes an error code instead of a stray access.

Each case runs in a child process that selects the checked build before loading the library
(a process holds one build). It checks the checked build against the oracle on valid input,
then corrupts the router's CSR in three ways and checks the reported code, and after each
corruption routes again on the same stream and checks that the attention is bit for bit the
first valid output."""
import json
import os
import subprocess
import sys
import textwrap

import pytest
import torch

from block_sparse_top_fvattn_b200 import _lib

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent(r"""
    import json, sys
    import numpy as np
    import torch
    sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
    from block_sparse_top_fvattn_b200 import _lib
    _lib.use_debug_build()
    import block_sparse_top_fvattn_b200 as fv
    from test_gpu_parity import check_route, check_attention, small_inputs, MAX_ABS_F32
    lib = fv.load()
    out = {{"lib": lib._name}}
    dtype = {dtype!r}
    if dtype == "bf16":
        w, q, k, v = small_inputs("single", H=3, S=2500)
        tol = {{}}
        cfg = fv.RouteConfig(p=0.9)
    else:
        w, q, k, v = small_inputs("tiny")
        tol = dict(max_abs=MAX_ABS_F32, mean_abs=MAX_ABS_F32)
        cfg = fv.RouteConfig(p=0.9, local_window=1)           # rows of at least two blocks
    scale = 1.0 / np.sqrt(w.d)
    csr, gm, r = check_route(q, k, cfg)
    check_attention(q, k, v, csr, r, gm, scale, **tol)        # the checked build against the oracle
    o_ref = fv.sparse_attn(q, k, v, csr).clone()
    rp = csr.row_ptr.cpu().numpy()
    nb = csr.nb
    row = int(np.argmax(np.diff(rp)))                          # a row with the longest list
    assert rp[row + 1] - rp[row] >= 2
    def corrupt(kind):
        if kind == "column":
            csr.col_idx[int(rp[row])] = nb + 3
        elif kind == "offsets":                                # rows `row` and row + 1 both fail
            csr.row_ptr[row + 1] = csr.col_idx.numel() + 5
        else:
            a = int(rp[row])
            x0, x1 = int(csr.col_idx[a]), int(csr.col_idx[a + 1])
            csr.col_idx[a], csr.col_idx[a + 1] = x1, x0
    res = {{}}
    for kind in ("column", "offsets", "order"):
        corrupt(kind)
        o = torch.full_like(q, 7.0)
        fv.sparse_attn(q, k, v, csr, out=o)
        st = fv.read_status(csr)
        detail = int(csr.status[1].item())
        # route again on the same stream: the CSR is rewritten and the status reset
        fv.route(q, k, cfg, csr=csr)
        o2 = fv.sparse_attn(q, k, v, csr)
        res[kind] = [st, detail, fv.read_status(csr), bool(torch.equal(o2, o_ref))]
    out["cases"] = res
    print("RESULT " + json.dumps(out))
""")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    if not os.path.exists(_lib.DEBUG_LIB_PATH):
        pytest.fail(f"{_lib.DEBUG_LIB_PATH} is missing; build it with `python -m block_sparse_top_fvattn_b200.build --debug`")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_checked_build_parity_and_corrupt_csr(dtype):
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"), dtype=dtype)
    p = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stdout[-3000:] + p.stderr[-3000:]
    line = [x for x in p.stdout.splitlines() if x.startswith("RESULT ")][-1]
    res = json.loads(line[len("RESULT "):])
    assert res["lib"].endswith("libfvattn_debug.so")
    want = {"column": _lib.DEBUG_COLUMN, "offsets": _lib.DEBUG_OFFSETS, "order": _lib.DEBUG_ORDER}
    for kind, (st, detail, st_after, same) in res["cases"].items():
        assert st == _lib.FVATTN_ERR_INVALID, (kind, st)
        assert detail == want[kind], (kind, detail)
        assert st_after == _lib.FVATTN_OK, (kind, st_after)
        assert same, kind
