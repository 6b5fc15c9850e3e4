"""Pins for the oracle's decoder-stack forward and layer-wise scores.

Each pin reaches its expected value without the oracle's own code path:
closed forms (RMSNorm's mean square, one rotary pair by hand, one-token
attention), invariants (rotary relative positions, causality, grouped heads)
and degenerate weights (a zero stack is the final norm of its input; a zero
layer quantises to zero and scores 0).
"""
import math

import numpy as np
import pytest

import oracle
from oracle import stack
from tests import brute

CFG = stack.StackConfig(hidden=64, n_heads=4, n_kv_heads=2, mlp=96, rope_theta=10000.0)


def _blocks(rng, n, cfg=CFG, std=0.05):
    d = cfg.head_dim
    shapes = [(cfg.n_heads * d, cfg.hidden), (cfg.n_kv_heads * d, cfg.hidden), (cfg.n_kv_heads * d, cfg.hidden),
              (cfg.hidden, cfg.n_heads * d), (cfg.mlp, cfg.hidden), (cfg.mlp, cfg.hidden), (cfg.hidden, cfg.mlp)]
    return [tuple(rng.normal(0, std, s) for s in shapes) for _ in range(n)]


def test_rms_norm_mean_square():
    rng = np.random.default_rng(0)
    x = rng.normal(0, 3, (5, 64))
    y = stack.rms_norm(x, 1e-5)
    ms = np.mean(x * x, axis=1)
    assert np.allclose(np.mean(y * y, axis=1), ms / (ms + 1e-5), rtol=1e-14)


def test_rope_by_hand_and_relative_positions():
    d, theta = 16, 10000.0
    x = np.zeros((4, d))
    x[:, 0] = 1.0                                     # unit vector on pair (0, d/2)
    x[:, 3] = 2.0                                     # pair (3, d/2 + 3)
    y = stack.rope(x, 1, theta)
    for t in range(4):
        assert math.isclose(y[t, 0], math.cos(t), abs_tol=1e-15)
        assert math.isclose(y[t, d // 2], math.sin(t), abs_tol=1e-15)
        a = t * theta ** (-6.0 / d)
        assert math.isclose(y[t, 3], 2 * math.cos(a), abs_tol=1e-15)
        assert math.isclose(y[t, d // 2 + 3], 2 * math.sin(a), abs_tol=1e-15)
    # <rope(q)_m, rope(k)_n> depends on m - n only
    rng = np.random.default_rng(1)
    q1, k1 = rng.normal(size=d), rng.normal(size=d)
    Q = stack.rope(np.tile(q1, (9, 1)), 1, theta)
    Kr = stack.rope(np.tile(k1, (9, 1)), 1, theta)
    assert math.isclose(Q[5] @ Kr[2], Q[8] @ Kr[5], rel_tol=1e-12)
    assert np.allclose(np.linalg.norm(Q, axis=1), np.linalg.norm(q1), rtol=1e-14)


def test_attention_one_token_and_grouping():
    rng = np.random.default_rng(2)
    T, H, G, d = 1, 4, 2, 8
    q, k, v = rng.normal(size=(T, H * d)), rng.normal(size=(T, G * d)), rng.normal(size=(T, G * d))
    out = stack.causal_attention(q, k, v, H, G)
    for h in range(H):                                 # one key: the output is its value, head h on kv head h // 2
        assert np.array_equal(out[0, h * d:(h + 1) * d], v[0, (h // 2) * d:(h // 2 + 1) * d])


def test_attention_is_causal():
    rng = np.random.default_rng(3)
    T, H, G, d = 6, 2, 1, 8
    q, k, v = rng.normal(size=(T, H * d)), rng.normal(size=(T, G * d)), rng.normal(size=(T, G * d))
    a = stack.causal_attention(q, k, v, H, G)
    k2, v2 = k.copy(), v.copy()
    k2[4:] += 10.0
    v2[4:] -= 3.0
    b = stack.causal_attention(q, k2, v2, H, G)
    assert np.array_equal(a[:4], b[:4]) and not np.allclose(a[4:], b[4:])
    # two steps by hand at t = 1 for head 0: weights softmax(q1.k0, q1.k1) / sqrt(d)
    s = np.array([q[1, :d] @ k[0], q[1, :d] @ k[1]]) / math.sqrt(d)
    p = np.exp(s - s.max()) / np.exp(s - s.max()).sum()
    assert np.allclose(a[1, :d], p[0] * v[0] + p[1] * v[1], rtol=1e-13)


def test_zero_stack_is_the_norm_of_its_input():
    rng = np.random.default_rng(4)
    x = rng.normal(0, 2, (5, 64))
    blocks = [tuple(np.zeros_like(w) for w in Ws) for Ws in _blocks(rng, 2)]
    assert np.allclose(stack.stack_output(x, blocks, CFG), x / np.sqrt(np.mean(x * x, 1, keepdims=True) + 1e-5),
                       rtol=1e-14)
    assert np.all(stack.layer_scores(x, blocks, CFG) == 0.0)


def test_zero_layer_scores_zero_and_others_positive():
    rng = np.random.default_rng(5)
    x = rng.normal(0, 1, (6, 64))
    blocks = _blocks(rng, 2)
    b1 = list(blocks[1])
    b1[4] = np.zeros_like(b1[4])                       # block 1's gate is zero
    blocks[1] = tuple(b1)
    sc = stack.layer_scores(x, blocks, CFG)
    assert sc.shape == (14,)
    # a zero gate zeroes the block's MLP product, so gate, up and down of that
    # block all leave the output unchanged when quantised
    assert np.all(sc[[11, 12, 13]] == 0.0) and np.all(sc[:11] > 0.0)


def test_quantized_linear_is_the_bf16_of_the_decoded_product():
    rng = np.random.default_rng(6)
    x, W = rng.normal(size=(3, 64)), rng.normal(0, 0.05, (5, 64))
    y = stack.quantized_linear(x, W)
    ac, as_ = oracle.quantize_rows(x, None, (0, 0, 64))
    wc, ws = oracle.quantize_rows(W, None, (0, 0, 64))
    xa = brute.to_f64(brute.decode_rows(ac, as_, (0, 0, 64)))
    wa = brute.to_f64(brute.decode_rows(wc, ws, (0, 0, 64)))
    exact = xa @ wa.T
    assert np.all(np.abs(y - exact) <= np.abs(exact) * 2.0 ** -9)   # within half a bf16 step
    # bf16 values have 8 significant bits
    m, _ = np.frexp(y)
    assert np.array_equal(m * 256, np.rint(m * 256))


@pytest.mark.parametrize("v,want", [(1.0 + 2 ** -9, 1.0), (1.0 + 3 * 2 ** -9, 1.0 + 2 ** -7),
                                    (-(1.0 + 2 ** -8), -1.0), (-(1.0 + 2 ** -7), -(1.0 + 2 ** -7)), (3.0 * 2 ** -140, 3.0 * 2 ** -140)])
def test_round_bf16_ties_to_even(v, want):
    assert stack.round_bf16(np.array([v]))[0] == want
