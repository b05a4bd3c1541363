"""The failure path of the bounded device waits, run on purpose without a GPU fault.

Every barrier wait of the tensor-core kernels is bounded. fvattn_sparse_attn_timeout_check and
fvattn_block_scores_timeout_check make each CTA first wait on a barrier that nothing completes,
with a short poll limit and before any copy or MMA: the wait runs out, every role of the CTA
unwinds, tensor memory is freed and FVATTN_ERR_TIMEOUT lands in the device status word. The
tests check that status, that no output was written, and that the same stream then runs the
normal calls with results equal to the oracle's."""
import numpy as np
import pytest
import torch

import block_sparse_top_fvattn_b200 as fv
from block_sparse_top_fvattn_b200 import _lib
from test_gpu_parity import check_attention, check_route, small_inputs
from test_gpu_scores import test_block_scores_match_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fv.load()


@pytest.mark.parametrize("polls", [1, 64])
def test_attention_wait_runs_out_then_stream_is_usable(polls):
    w, q, k, v = small_inputs("single", H=3, S=2500)
    cfg = fv.RouteConfig(p=0.9)
    csr, gm, r = check_route(q, k, cfg)
    out = torch.full_like(q, 3.0)
    st = fv.sparse_attn_timeout_check(q, k, v, csr, out, polls=polls)
    assert st == _lib.FVATTN_ERR_TIMEOUT
    assert int(csr.status[1].item()) == 20                     # the scheduler's first wait
    assert bool((out == 3.0).all())                            # nothing written
    # the stream and the context stay usable: route again (resets the status) and attend
    csr, gm, r = check_route(q, k, cfg, csr=csr)
    check_attention(q, k, v, csr, r, gm, 1.0 / np.sqrt(w.d))


def test_attention_timeout_check_rejects_bad_arguments():
    w, q, k, v = small_inputs("single", H=1, S=256)
    csr = fv.route(q, k, fv.RouteConfig(p=0.9))
    with pytest.raises(fv.FvattnError) as e:
        fv.sparse_attn_timeout_check(q, k, v, csr, torch.empty_like(q), polls=0)
    assert e.value.code == _lib.FVATTN_ERR_INVALID
    w, qf, kf, vf = small_inputs("tiny")                       # fp32: no tensor-core kernel
    csr = fv.route(qf, kf, fv.RouteConfig(p=0.9))
    with pytest.raises(fv.FvattnError) as e:
        fv.sparse_attn_timeout_check(qf, kf, vf, csr, torch.empty_like(qf), polls=4)
    assert e.value.code == _lib.FVATTN_ERR_UNSUPPORTED


@pytest.mark.parametrize("polls", [1, 64])
def test_score_wait_runs_out_then_stream_is_usable(polls):
    w, q, k, _ = small_inputs("single", H=2, S=3000)
    st, out = fv.block_scores_timeout_check(q, k, polls=polls)
    assert st == _lib.FVATTN_ERR_TIMEOUT
    assert bool(torch.isnan(out).all())                        # no score written
    # the normal call on the same stream still matches the oracle element by element
    test_block_scores_match_oracle("single", dict(H=2, S=3000))
