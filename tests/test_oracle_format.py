"""Pins for the oracle's MXINT block format (codes, exponent, packing).

Each check reaches the expected value by a route other than the oracle's:
hand-derived golden blocks, brute-force nearest-grid search, exact
comparisons with powers of two, and closed-form invariants of the format.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "format_blocks.json")


def _blocks(seed, n=64):
    """Random blocks: normal, heavy-tailed, tiny (fp32 subnormal), huge, exact ties."""
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        kind = i % 6
        if kind == 0:
            b = rng.normal(0, 1, 32)
        elif kind == 1:
            b = rng.standard_t(3, 32) * 0.02
            b[rng.integers(32)] *= 50
        elif kind == 2:
            b = rng.normal(0, 1, 32) * 1e-40          # fp32 subnormal range
        elif kind == 3:
            b = rng.normal(0, 1, 32) * 1e37
        elif kind == 4:                               # exact half-step ties
            e = int(rng.integers(-10, 10))
            b = (rng.integers(-60, 60, 32) + 0.5) * 2.0 ** (e - 6)
            b[0] = 2.0 ** e * 1.5
        else:
            b = rng.normal(0, 1, 32)
            b[rng.integers(0, 32, 5)] = 0.0
        out.append(np.asarray(b, dtype=np.float32).astype(np.float64))
    return out


def test_golden_blocks():
    cases = json.load(open(GOLDEN))["cases"]
    for case in cases:
        x = np.zeros(32)
        x[:len(case["x"])] = case["x"]
        for m_str, expect in case["codes"].items():
            m = int(m_str)
            q, e = oracle.quant_block(x, m)
            assert e + 127 == case["scale_byte"], case["name"]
            assert list(q[:len(expect)]) == expect, (case["name"], m)
            assert not np.any(q[len(expect):]), case["name"]
        for m_str, prefix in case.get("packed_prefix", {}).items():
            m = int(m_str)
            q, _ = oracle.quant_block(x, m)
            packed = oracle.pack(q, m)
            assert [int(h, 16) for h in prefix] == list(packed[:len(prefix)]), (case["name"], m)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_exponent_brackets_block_max(seed):
    for b in _blocks(seed):
        e = oracle.block_exp(b)
        assert e == brute.exact_exponent(b)
        amax = float(np.max(np.abs(b)))
        if amax >= 2.0 ** -127:
            assert math.ldexp(1.0, e) <= amax < math.ldexp(1.0, e + 1)


@pytest.mark.parametrize("m", [4, 6, 8])
@pytest.mark.parametrize("seed", [0, 1])
def test_codes_match_nearest_grid_search(m, seed):
    for b in _blocks(seed + 10 * m, n=24):
        q, e = oracle.quant_block(b, m)
        bq, be = brute.brute_block(b, m)
        assert e == be
        assert list(q) == bq


@pytest.mark.parametrize("m", [4, 6, 8])
def test_invariants(m):
    L = (1 << (m - 1)) - 1
    for b in _blocks(7 + m):
        q, e = oracle.quant_block(b, m)
        step = math.ldexp(1.0, e - m + 2)
        deq = oracle.dequant(q, e, m)
        # (i) idempotence: re-quantising the dequantised block changes nothing
        q2, e2 = oracle.quant_block(deq, m)
        if np.any(q):
            assert e2 == e and np.array_equal(q2, q)
        # (ii) per-element error <= step/2 unless the code is at the clamp
        err = np.abs(b - deq)
        inside = np.abs(q) < L
        if np.max(np.abs(b)) >= 2.0 ** -127:
            assert np.all(err[inside] <= step / 2 * (1 + 1e-15))
            # block max is within one step of its code
            j = int(np.argmax(np.abs(b)))
            assert abs(abs(b[j]) - abs(deq[j])) <= step
        assert np.all(np.abs(q) <= L)


def test_error_nests_by_width():
    for b in _blocks(99, n=120):
        errs = []
        for m in (8, 6, 4):
            q, e = oracle.quant_block(b, m)
            errs.append(np.abs(b - oracle.dequant(q, e, m)))
        assert np.all(errs[0] <= errs[1]) and np.all(errs[1] <= errs[2])
        assert errs[0].dot(errs[0]) <= errs[1].dot(errs[1]) <= errs[2].dot(errs[2])


@pytest.mark.parametrize("m", [4, 6, 8])
def test_exact_round_trip_sets(m):
    rng = np.random.default_rng(m)
    L = (1 << (m - 1)) - 1
    for _ in range(50):
        e = int(rng.integers(-120, 120))
        codes = rng.integers(-L, L + 1, 32)
        codes[0] = int(rng.choice([-1, 1])) * int(rng.integers(1 << (m - 2), L + 1))
        x = np.array([math.ldexp(float(c), e - m + 2) for c in codes])
        q, e2 = oracle.quant_block(x, m)
        assert e2 == e
        assert np.array_equal(q, codes)
        assert np.array_equal(oracle.dequant(q, e2, m), x)
    # all-equal +-2^k blocks round-trip exactly ...
    for k in (-100, -3, 0, 5, 100):
        for sgn in (1.0, -1.0):
            x = np.full(32, sgn * 2.0 ** k)
            q, e = oracle.quant_block(x, m)
            assert np.array_equal(oracle.dequant(q, e, m), x)
    # ... but an all-equal block is NOT exact in general: 1.1 is off the grid.
    x = np.full(32, 1.1)
    q, e = oracle.quant_block(x, m)
    assert not np.array_equal(oracle.dequant(q, e, m), x)


@pytest.mark.parametrize("m", [4, 6, 8])
def test_pack_unpack_all_codes(m):
    L = (1 << (m - 1)) - 1
    codes = np.array(list(range(-L, L + 1)) * 4, dtype=np.int32)
    codes = codes[:len(codes) // 32 * 32]
    packed = oracle.pack(codes, m)
    assert bytes(packed) == brute.pack_bits(codes, m)
    assert np.array_equal(oracle.unpack(packed, codes.size, m), codes)
    assert brute.unpack_bits(bytes(packed), codes.size, m) == list(codes)


def test_dequant_values_exact():
    for m in (4, 6, 8):
        for e in (-127, -60, 0, 60, 127):
            for c in (-(1 << (m - 1)) + 1, -1, 0, 1, (1 << (m - 1)) - 1):
                v = oracle.dequant(np.array([c]), e, m)[0]
                assert Fraction(v) == brute.code_value(c, e, m)
