"""Pins for the oracle's decode-step attention over MXINT4 K/V caches.

The caches are built here code by code (pure-Python bit packing) and decoded
independently (pure-Python unpacking, exact fractions), so each pin reaches
the expected output by a route that shares nothing with the oracle:
  - one token: the output is that token's decoded value row, exactly;
  - zero query (or zero scale): uniform weights, the exact mean of the
    group's value rows; with two kv heads this also pins the head grouping;
  - two tokens: the closed form p = 1 / (1 + e^(s1 - s0)) on hand-made codes;
  - a value scale byte one higher doubles the output exactly;
  - reordering the tokens (K and V together) leaves the output unchanged;
  - one dominant score selects its token's values.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests import brute


def _cache_rows(code_rows, scale_rows):
    """Compact (rows x d/2, rows x d/32) uint8 arrays from per-row code lists
    and per-row scale-byte lists (4-bit codes, blocks of 32)."""
    codes = np.array([list(brute.pack_bits(c, 4)) for c in code_rows], dtype=np.uint8)
    scales = np.array(scale_rows, dtype=np.uint8)
    return codes, scales


def _decode(codes, scales):
    return brute.decode_rows([np.zeros((codes.shape[0], 0), np.uint8)] * 2 + [codes],
                             [np.zeros((codes.shape[0], 0), np.uint8)] * 2 + [scales], [0, 0, codes.shape[1] * 2])


def _random_cache(rng, rows, d):
    code_rows = [list(rng.integers(-7, 8, d)) for _ in range(rows)]
    scale_rows = [list(rng.integers(120, 131, d // 32)) for _ in range(rows)]
    return _cache_rows(code_rows, scale_rows)


def test_single_token_returns_its_values():
    rng = np.random.default_rng(0)
    d, n_kvh, n_qh = 64, 2, 4
    kc, ks = _random_cache(rng, n_kvh, d)
    vc, vs = _random_cache(rng, n_kvh, d)
    q = rng.normal(0, 1, (n_qh, d))
    out = oracle.attn_decode(q, kc, ks, vc, vs, 1, n_kvh, 0.125)
    vdec = brute.to_f64(_decode(vc, vs))
    for h in range(n_qh):
        assert np.array_equal(out[h], vdec[h // 2])


@pytest.mark.parametrize("how", ["zero_query", "zero_scale"])
def test_uniform_weights_give_the_group_mean(how):
    rng = np.random.default_rng(1)
    d, n_kvh, n_qh, T = 32, 2, 4, 8
    kc, ks = _random_cache(rng, T * n_kvh, d)
    vc, vs = _random_cache(rng, T * n_kvh, d)
    q = np.zeros((n_qh, d)) if how == "zero_query" else rng.normal(0, 1, (n_qh, d))
    out = oracle.attn_decode(q, kc, ks, vc, vs, T, n_kvh, 0.0 if how == "zero_scale" else 0.5)
    vdec = _decode(vc, vs)
    for h in range(n_qh):
        g = h // (n_qh // n_kvh)                    # heads 0, 1 -> kv head 0; 2, 3 -> kv head 1
        mean = [sum(vdec[t * n_kvh + g, i] for t in range(T)) / T for i in range(d)]
        assert np.array_equal(out[h], np.array([float(x) for x in mean]))


def test_two_tokens_closed_form():
    d = 32
    # K: token 0 codes all +1, token 1 all -2, scale byte 127 (e = 0, step 2^-2)
    kc, ks = _cache_rows([[1] * d, [-2] * d], [[127], [127]])
    # V: token 0 codes all +3, token 1 all -4
    vc, vs = _cache_rows([[3] * d, [-4] * d], [[127], [127]])
    q = np.ones((1, d))
    out = oracle.attn_decode(q, kc, ks, vc, vs, 2, 1, 0.125)
    s0, s1 = 0.125 * 32 * 0.25, 0.125 * 32 * -0.5          # 1 and -2
    p0 = 1.0 / (1.0 + math.exp(s1 - s0))
    want = p0 * 0.75 + (1.0 - p0) * -1.0
    assert np.allclose(out, want, rtol=1e-15, atol=0)


def test_value_scale_doubles_output():
    rng = np.random.default_rng(2)
    d, T = 64, 16
    kc, ks = _random_cache(rng, T, d)
    vc, vs = _random_cache(rng, T, d)
    q = rng.normal(0, 1, (2, d))
    a = oracle.attn_decode(q, kc, ks, vc, vs, T, 1, 0.3)
    b = oracle.attn_decode(q, kc, ks, vc, vs + 1, T, 1, 0.3)
    assert np.array_equal(b, 2.0 * a)


def test_token_order_does_not_matter():
    rng = np.random.default_rng(3)
    d, T, n_kvh = 64, 37, 2
    kc, ks = _random_cache(rng, T * n_kvh, d)
    vc, vs = _random_cache(rng, T * n_kvh, d)
    q = rng.normal(0, 1, (4, d))
    a = oracle.attn_decode(q, kc, ks, vc, vs, T, n_kvh, 0.2)
    perm = rng.permutation(T)
    rows = (perm[:, None] * n_kvh + np.arange(n_kvh)[None, :]).ravel()
    b = oracle.attn_decode(q, kc[rows], ks[rows], vc[rows], vs[rows], T, n_kvh, 0.2)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-15)


def test_dominant_score_selects_its_token():
    rng = np.random.default_rng(4)
    d, T = 32, 10
    code_rows = [[0] * d for _ in range(T)]
    code_rows[6] = [7] * d                              # s_6 = 32 * 7 * 0.25 * 4 = 224, others 0
    kc, ks = _cache_rows(code_rows, [[127]] * T)
    vc, vs = _random_cache(rng, T, d)
    out = oracle.attn_decode(np.full((1, d), 4.0), kc, ks, vc, vs, T, 1, 1.0)
    v6 = brute.to_f64(_decode(vc, vs))[6]
    assert np.allclose(out[0], v6, rtol=0, atol=1e-90)
    assert Fraction(1) / (1 + 9 * Fraction(math.exp(-224))) > 1 - Fraction(1, 10 ** 90)
