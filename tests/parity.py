"""Shared helpers of the GPU parity tests: run the same seeded inputs through
the CUDA library (via the C ABI binding) and through the CPU oracle, and
compare.  The oracle always reads back the exact bytes the GPU consumed."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle

GEMM_TOL = 2e-3          # relative error budget of mxs_gemm beyond the bf16 output rounding
GEMM_FLOOR = 1e-2        # relative-error denominator floor, as a fraction of max|Yref|
# normwise bound: the arithmetic budget plus the bf16 output rounding (8
# significant bits: at most 2^-8 of the unrounded value's magnitude)
GEMM_NORMWISE_TOL = GEMM_TOL + 2.0 ** -8 * (1.0 + GEMM_TOL)


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    major, _ = torch.cuda.get_device_capability()
    if major != 10:
        pytest.skip("needs an sm_100 device")


def capi():
    from mx_microscaling_mixed_b200 import build
    build.build()
    from mx_microscaling_mixed_b200 import capi as c
    return c


def host64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def compact(t, g):
    return t.code_rows(g).cpu().numpy(), t.scale_rows(g).cpu().numpy()


def assert_codes_equal(gpu_t, o_codes, o_scales, what=""):
    for g in range(3):
        c, s = compact(gpu_t, g)
        assert c.shape == o_codes[g].shape and s.shape == o_scales[g].shape, (what, g)
        bad = np.argwhere(c != o_codes[g])
        assert bad.size == 0, f"{what} seg {g}: {bad.shape[0]} code bytes differ, first {bad[:3].tolist()}"
        bad = np.argwhere(s != o_scales[g])
        assert bad.size == 0, f"{what} seg {g}: {bad.shape[0]} scale bytes differ, first {bad[:3].tolist()}"


def half_ulp_bf16(x: np.ndarray) -> np.ndarray:
    """Half a bf16 unit in the last place at |x| (8 significant bits)."""
    _, ex = np.frexp(np.abs(x))          # |x| = f 2^ex, f in [0.5, 1)
    return np.where(x == 0, 0.0, np.ldexp(1.0, ex - 9))


def gemm_rel_error(Y: np.ndarray, Yref: np.ndarray) -> float:
    """Relative error of bf16 Y against the fp64 product Yref, beyond the
    output rounding: max over elements of
        max(0, |Y - Yref| - half_ulp_bf16(max(|Y|, |Yref|))) / max(|Yref|, 1% max|Yref|).
    bf16 keeps 8 significant bits, so rounding the exact result alone moves
    it by up to 2^-8 = 3.9e-3 relative; the 2e-3 budget applies to the
    arithmetic before that rounding (fp32 accumulation)."""
    ymax = float(np.max(np.abs(Yref))) if Yref.size else 0.0
    if ymax == 0.0:
        return float(np.max(np.abs(Y))) if Y.size else 0.0
    den = np.maximum(np.abs(Yref), GEMM_FLOOR * ymax)
    excess = np.maximum(0.0, np.abs(Y - Yref) - half_ulp_bf16(np.maximum(np.abs(Y), np.abs(Yref))))
    return float(np.max(excess / den))


def gemm_normwise_error(Y: np.ndarray, Yref: np.ndarray) -> float:
    """Normwise error max|Y - Yref| / max|Yref|, output rounding included
    (0 when both are all zero)."""
    ymax = float(np.max(np.abs(Yref))) if Yref.size else 0.0
    diff = float(np.max(np.abs(Y - Yref))) if Y.size else 0.0
    return diff / ymax if ymax > 0.0 else diff


def quantize_both(c, src: torch.Tensor, layout, perm_np, counts, weight: bool):
    """GPU MXTensor and the oracle's compact (codes, scales) for the same bytes."""
    t = c.mxtensor_empty(src.shape[0], layout, device=src.device)
    (c.mxs_quantize_weight if weight else c.mxs_quantize_act)(src, t)
    oc, os_ = oracle.quantize_rows(host64(src), perm_np, counts)
    return t, oc, os_
