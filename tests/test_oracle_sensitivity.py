"""Pins for the oracle's column sensitivity (H diagonal, Q4 error, s = H * E).

Expected values come from exact rational arithmetic on the same inputs
(fractions.Fraction), with Q4 computed by brute-force nearest-grid search,
plus closed-form special cases.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests import brute


def _exact_sensitivity(X, W):
    T, K = X.shape
    N = W.shape[0]
    H = [Fraction(2) * sum(Fraction(float(X[t, j])) ** 2 for t in range(T)) / T for j in range(K)]
    E = [Fraction(0)] * K
    for i in range(N):
        for b0 in range(0, K, 32):
            blk = [float(W[i, j]) if j < K else 0.0 for j in range(b0, b0 + 32)]
            q, e = brute.brute_block(blk, 4)
            for t in range(32):
                j = b0 + t
                if j < K:
                    E[j] += (Fraction(blk[t]) - brute.code_value(q[t], e, 4)) ** 2
    return H, E


def _close(a, exact, terms):
    """fp64 value within terms * 2^-52 relative of the exact rational."""
    if exact == 0:
        return a == 0.0
    return abs(Fraction(a) - exact) <= abs(exact) * Fraction(terms + 2, 2 ** 52)


@pytest.mark.parametrize("T,N,K,seed", [(5, 3, 32, 0), (8, 8, 40, 1), (150, 70, 45, 2)])
def test_matches_exact_rationals(T, N, K, seed):
    rng = np.random.default_rng(seed)
    X = rng.normal(0, 1, (T, K)).astype(np.float32)
    X[:, rng.integers(0, K, 3)] *= 30
    W = (rng.normal(0, 0.02, (N, K)) * (1 + 20 * (rng.random(K) < 0.1))).astype(np.float32)
    H, E, s = oracle.sensitivity(X, W)
    He, Ee = _exact_sensitivity(X, W)
    for j in range(K):
        assert _close(H[j], He[j], T), j
        assert _close(E[j], Ee[j], N), j
        assert _close(s[j], He[j] * Ee[j], T + N + 1), j


def test_bf16_inputs_exact_squares():
    import torch
    g = torch.Generator().manual_seed(3)
    X = torch.randn(70, 33, generator=g).to(torch.bfloat16).float().numpy()
    W = (torch.randn(9, 33, generator=g) * 0.02).to(torch.bfloat16).float().numpy()
    H, E, s = oracle.sensitivity(X, W)
    He, Ee = _exact_sensitivity(X, W)
    for j in range(33):
        assert _close(H[j], He[j], 70) and _close(E[j], Ee[j], 9)


def test_ones_column_gives_two():
    X = np.random.default_rng(0).normal(0, 1, (100, 64))
    X[:, 5] = 1.0
    H, _, _ = oracle.sensitivity(X.astype(np.float32), np.ones((4, 64), np.float32))
    assert H[5] == 2.0


def test_grid_weights_have_zero_error():
    rng = np.random.default_rng(1)
    # every block of every row lies on its own 4-bit grid -> Q4 is exact
    W = np.zeros((6, 96))
    for i in range(6):
        for b in range(3):
            e = int(rng.integers(-8, 3))
            codes = rng.integers(-7, 8, 32)
            codes[0] = 5
            W[i, 32 * b:32 * b + 32] = codes * 2.0 ** (e - 2)
    X = rng.normal(0, 1, (10, 96))
    H, E, s = oracle.sensitivity(X.astype(np.float32), W.astype(np.float32))
    assert np.all(E == 0.0) and np.all(s == 0.0) and np.all(H > 0)


def test_scaling_column_scales_h_quadratically():
    rng = np.random.default_rng(2)
    X = rng.normal(0, 1, (64, 32)).astype(np.float32)
    X2 = X.copy()
    X2[:, 7] *= 4.0
    W = rng.normal(0, 1, (3, 32)).astype(np.float32)
    H1, _, _ = oracle.sensitivity(X, W)
    H2, _, _ = oracle.sensitivity(X2, W)
    assert H2[7] == 16.0 * H1[7]
    assert np.array_equal(np.delete(H1, 7), np.delete(H2, 7))


def test_short_last_block_is_zero_padded():
    # K = 33: column 32 forms a block of its own, padded with zeros; its Q4
    # uses its own exponent, not that of columns 0..31.
    W = np.zeros((1, 33), np.float32)
    W[0, :32] = 100.0
    W[0, 32] = 0.3
    X = np.ones((2, 33), np.float32)
    _, E, _ = oracle.sensitivity(X, W)
    # 0.3 alone: e = -2, step 2^-4, code round(4.8) = 5 -> error (0.3 - 5/16)^2
    assert E[32] == pytest.approx((np.float64(np.float32(0.3)) - 5 / 16) ** 2, rel=1e-15)
