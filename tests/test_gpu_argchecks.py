"""GPU: argument checks that can be made with real device buffers.

Each call below is wrong in its shape relations only, and every buffer is
large enough that even a call whose check failed to reject it would stay
inside its allocations; the library must return the status before any launch
(the launch counter does not move)."""
import ctypes

import pytest
import torch

from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def c():
    parity.need_gpu()
    return parity.capi()


def _status(fn):
    try:
        fn()
    except parity.capi().MxsError as e:
        return e.status
    return 0


def test_gemm_shape_checks(c):
    # K = 250: layouts (30, 60, 160) and (28, 62, 160) pad to the same
    # (32, 64, 160) positions but are different layouts
    la = c.mxs_layout_make(250, (30, 60, 160), torch.arange(250, dtype=torch.int32, device="cuda"))
    lb = c.mxs_layout_make(250, (28, 62, 160), la.perm)
    A, W, W2 = c.mxtensor_empty(64, la), c.mxtensor_empty(96, la), c.mxtensor_empty(96, lb)
    Y = torch.zeros(64, 96, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(c.mxs_gemm_workspace_bytes(A, W) + 4096, dtype=torch.uint8, device="cuda")
    n0 = c.mxs_launch_count()
    assert _status(lambda: c.mxs_gemm(A, W2, Y=Y, workspace=ws)) == 2            # layouts differ
    st = c._lib.mxs_gemm(ctypes.byref(A.c), ctypes.byref(W.c), Y.data_ptr(), 95, c._aligned_ptr(ws),
                         ws.numel() - 1024, None)
    assert st == 2                                                                   # ldy < N
    assert c.mxs_launch_count() == n0


def test_quantize_and_sensitivity_shape_checks(c):
    lay = c.mxs_layout_make(64, (0, 0, 64))
    t = c.mxtensor_empty(8, lay)
    src = torch.zeros(8, 64, dtype=torch.bfloat16, device="cuda")
    n0 = c.mxs_launch_count()
    # fewer rows than the output holds -> MXS_ERR_SHAPE
    assert c._lib.mxs_quantize_act(src.data_ptr(), 1, 7, 64, ctypes.byref(t.c), None) == 2
    # pitch below K
    assert c._lib.mxs_quantize_weight(src.data_ptr(), 1, 8, 63, ctypes.byref(t.c), None) == 2
    X = torch.zeros(128, 512, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(256, 512, dtype=torch.bfloat16, device="cuda")
    H, E, S = (torch.empty(512, dtype=torch.float64, device="cuda") for _ in range(3))
    need = c.mxs_sensitivity_workspace_bytes(128, 256, 512)
    ws = torch.empty(need + 1024, dtype=torch.uint8, device="cuda")
    f = c._lib.mxs_sensitivity
    assert f(X.data_ptr(), 1, 128, 512, 511, W.data_ptr(), 1, 256, 512, H.data_ptr(), E.data_ptr(), S.data_ptr(),
             c._aligned_ptr(ws), need, None) == 2
    assert f(X.data_ptr(), 1, 128, 512, 512, W.data_ptr(), 1, 256, 512, H.data_ptr(), E.data_ptr(), S.data_ptr(),
             c._aligned_ptr(ws), need - 8, None) == 9
    assert c.mxs_launch_count() == n0
