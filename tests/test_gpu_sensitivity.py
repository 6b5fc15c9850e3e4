"""GPU parity: mxs_sensitivity (H diagonal, Q4 error, s) against the oracle,
bit for bit (both sum in the same pinned chunk order)."""
import numpy as np
import pytest
import torch

import oracle
from mx_microscaling_mixed_b200 import inputs
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def c():
    parity.need_gpu()
    return parity.capi()


def _check(c, X, W):
    H, E, s = c.mxs_sensitivity(X, W)
    torch.cuda.synchronize()
    Ho, Eo, so = oracle.sensitivity(parity.host64(X), parity.host64(W))
    for name, g, o in (("H", H, Ho), ("E", E, Eo), ("s", s, so)):
        g = g.cpu().numpy()
        bad = np.flatnonzero(g != o)
        assert bad.size == 0, f"{name}: {bad.size} columns differ, first {bad[:5]} {g[bad[:3]]} vs {o[bad[:3]]}"


def test_parity_layer(c):
    d = inputs.parity_layer("cuda", seed=0)
    _check(c, d["X"], d["W"])


@pytest.mark.parametrize("T,N,K,xd,wd", [
    (150, 70, 45, torch.float32, torch.float32),
    (150, 70, 45, torch.bfloat16, torch.float32),
    (65, 129, 264, torch.bfloat16, torch.bfloat16),
    (1, 1, 1, torch.float32, torch.bfloat16),
    (300, 40, 1000, torch.float32, torch.bfloat16),
    # TMA-tiled path: 16-byte aligned pitches, ragged chunk and column tile
    (130, 200, 1000, torch.bfloat16, torch.float32),
    (64, 64, 256, torch.float32, torch.float32),
    (257, 65, 4104, torch.bfloat16, torch.bfloat16),
    (3, 2, 8, torch.bfloat16, torch.bfloat16),
])
def test_ragged_shapes(c, T, N, K, xd, wd):
    X = inputs.random_matrix(T, K, device="cuda", seed=T, dtype=xd)
    W = inputs.random_matrix(N, K, device="cuda", seed=N + 1, dtype=wd, std=0.02)
    _check(c, X, W)


def test_strided_inputs(c):
    Xw = inputs.random_matrix(100, 203, device="cuda", seed=1, dtype=torch.bfloat16)
    Ww = inputs.random_matrix(77, 203, device="cuda", seed=2, dtype=torch.bfloat16)
    _check(c, Xw[:, :200], Ww[:, :200])    # pitch 203: not 16-byte aligned rows


def test_strided_aligned_inputs(c):
    Xw = inputs.random_matrix(100, 1032, device="cuda", seed=3, dtype=torch.bfloat16)
    Ww = inputs.random_matrix(90, 1040, device="cuda", seed=4, dtype=torch.float32)
    _check(c, Xw[:, :1000], Ww[:, :1000])    # 16-byte aligned pitches, ragged width


def test_tiny_and_zero_blocks(c):
    """Blocks whose maximum is below 2^-125 (the pre-scaled code path) and
    all-zero blocks, on the tiled and the streaming path."""
    for K in (512, 509):
        W = inputs.random_matrix(70, K, device="cuda", seed=5, dtype=torch.float32)
        W[:, 32:64] *= 2.0 ** -140
        W[3:9, 64:96] = 0.0
        W[10, :] *= 2.0 ** -128
        X = inputs.random_matrix(66, K, device="cuda", seed=6, dtype=torch.float32)
        _check(c, X, W)


def test_full_attention_layer(c):
    X = inputs.gaussian_acts("cuda", seed=2001, rows=2048, K=4096)
    W = inputs.attn_weight("cuda", seed=2000)
    _check(c, X, W)


def test_ones_column_is_two(c):
    X = torch.randn(100, 64, device="cuda")
    X[:, 5] = 1.0
    H, _, _ = c.mxs_sensitivity(X, torch.ones(4, 64, device="cuda"))
    assert H[5].item() == 2.0
