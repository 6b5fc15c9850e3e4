"""A device wait that runs out, without a fault: the prefill GEMM's
tensor-core kernels, given a spin limit of a few hundred nanoseconds by
mxs_set_wait_limit, give up in the middle of their pipelines.  Each CTA
records MXS_ERR_TIMEOUT in the status word, lets the copies and MMAs it had
already issued finish, frees its tensor memory and returns.  The host reads
the status through mxs_sync (once: the word is cleared), and the context
stays usable: at the default limit the same call matches the oracle."""
import numpy as np
import pytest
import torch

import oracle
from mx_microscaling_mixed_b200 import inputs
from tests import parity

pytestmark = pytest.mark.gpu

MXS_ERR_TIMEOUT = 7
SHORT_LIMIT = 1000        # SM cycles: far shorter than one output tile's main loop


@pytest.fixture(scope="module")
def c():
    parity.need_gpu()
    return parity.capi()


@pytest.mark.parametrize("M", [256, 1024])      # the one-CTA kernel; the 2-CTA pair kernel
def test_wait_expiry_reports_timeout_and_context_survives(c, M):
    N, K, counts = 2048, 32768, (32, 992, 31744)
    A = inputs.random_matrix(M, K, device="cuda", seed=M + 11, dtype=torch.bfloat16)
    W = inputs.random_matrix(N, K, device="cuda", seed=N + 13, dtype=torch.bfloat16, std=0.02)
    perm = np.random.default_rng(M).permutation(K).astype(np.int32)
    lay = c.mxs_layout_make(K, counts, torch.from_numpy(perm).cuda())
    Aq, Wq = c.mxtensor_empty(M, lay), c.mxtensor_empty(N, lay)
    c.mxs_quantize_act(A, Aq)
    c.mxs_quantize_weight(W, Wq)
    c.mxs_sync()
    assert c.mxs_gemm_workspace_bytes(Aq, Wq) > 0          # the tensor-core path, not the decode kernels

    c.mxs_set_wait_limit(SHORT_LIMIT)
    try:
        c.mxs_gemm(Aq, Wq)
        with pytest.raises(c.MxsError) as e:
            c.mxs_sync()
        assert e.value.status == MXS_ERR_TIMEOUT
    finally:
        c.mxs_set_wait_limit(0)
    c.mxs_sync()                                           # the word was cleared by the first read

    Y = c.mxs_gemm(Aq, Wq)
    c.mxs_sync()
    rows, cols = np.arange(0, M, 37), np.arange(0, N, 101)
    ac, as_ = oracle.quantize_rows(parity.host64(A[torch.from_numpy(rows).cuda()]), perm, counts)
    wc, ws = oracle.quantize_rows(parity.host64(W[torch.from_numpy(cols).cuda()]), perm, counts)
    Yref = oracle.gemm(ac, as_, wc, ws, counts)
    Yg = Y[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()].float().cpu().numpy().astype(np.float64)
    err = parity.gemm_rel_error(Yg, Yref)
    assert err <= parity.GEMM_TOL, f"max rel err {err:.3e}"
