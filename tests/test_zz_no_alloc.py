"""GPU: mxs_sensitivity_noalloc (fixed library scratch, no workspace) gives
the same bits as mxs_sensitivity, on two calls in a row through the C ABI,
and rejects shapes whose partials exceed the scratch before launching."""
import ctypes

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
    # (the scratch keeps the first call's partials: nothing may depend on them)
    shapes = [(2048, 4096, 4096, torch.bfloat16, torch.bfloat16, 2001),
              (130, 200, 1000, torch.bfloat16, torch.float32, 7)]
    for T, N, K, xd, wd, seed in shapes:
        X = inputs.random_matrix(T, K, device="cuda", seed=seed, dtype=xd)
        W = inputs.random_matrix(N, K, device="cuda", seed=seed + 1, dtype=wd, std=0.02)
        ref, got = _both(c, X, W)
        for name, r, g in zip("HEs", ref, got):
            assert torch.equal(r, g), name
    c.mxs_sync()


def test_too_large_is_rejected(c):
    # (ceil(T/64) + ceil(N/64)) * K * 8 bytes > 16 MiB
    T, N, K = 64, 64 * 1024, 4096
    need = c.mxs_sensitivity_workspace_bytes(T, N, K)
    assert need > c.NOALLOC_SCRATCH_BYTES
    launches = c.mxs_launch_count()
    d = lambda n: torch.empty(n, dtype=torch.float64, device="cuda")
    st = c._lib.mxs_sensitivity_noalloc(ctypes.c_void_p(1 << 20), 1, T, K, K, ctypes.c_void_p(1 << 21), 1, N, K,
                                        d(K).data_ptr(), d(K).data_ptr(), d(K).data_ptr(), None)
    assert st == 9                                    # MXS_ERR_WORKSPACE
    assert c.mxs_launch_count() == launches
