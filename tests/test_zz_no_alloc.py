"""GPU: mxs_sensitivity_noalloc (fixed library scratch, no workspace) gives
the same bits as mxs_sensitivity, on calls in a row through the C ABI.
Its rejection of shapes beyond the scratch is checked on the host
(tests/test_capi_host.py), where no launch can follow a failed check."""
import pytest
import torch

from mx_microscaling_mixed_b200 import inputs
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def c():
    parity.need_gpu()
    return parity.capi()


def _both(c, X, W):
    K = X.shape[1]
    ref = c.mxs_sensitivity(X, W)
    out = tuple(torch.full((K,), float("nan"), dtype=torch.float64, device="cuda") for _ in range(3))
    c.mxs_sensitivity_noalloc(X, W, out)
    torch.cuda.synchronize()
    return ref, out


def test_two_calls_match_workspace_entry(c):
    # first call: the attention-layer shape; second: a different, ragged one
    # (the scratch keeps the first call's partials: nothing may depend on
    # them); third: fp32 rows of 999 values, whose pitch is not a multiple of
    # 16 bytes, so the partials come from the register-streaming kernel,
    # which indexes the scratch its own way
    shapes = [(2048, 4096, 4096, torch.bfloat16, torch.bfloat16, 2001),
              (130, 200, 1000, torch.bfloat16, torch.float32, 7),
              (300, 170, 999, torch.float32, torch.float32, 11)]
    for T, N, K, xd, wd, seed in shapes:
        X = inputs.random_matrix(T, K, device="cuda", seed=seed, dtype=xd)
        W = inputs.random_matrix(N, K, device="cuda", seed=seed + 1, dtype=wd, std=0.02)
        ref, got = _both(c, X, W)
        for name, r, g in zip("HEs", ref, got):
            assert torch.equal(r, g), name
    c.mxs_sync()
