"""Pins for the oracle's row quantiser (permute, pad, code, pack) and GEMM.

The row quantiser is checked against a per-block brute-force quantiser run
on the gathered columns, decoded with pure-Python bit unpacking; the GEMM
against numpy's float64 matmul of independently decoded operands and
against closed-form special cases.
"""
import numpy as np
import pytest

import oracle
from tests import brute


def _layout(rng, K):
    n8 = int(rng.integers(0, K // 3 + 1))
    n6 = int(rng.integers(0, (K - n8) // 2 + 1))
    perm = rng.permutation(K).astype(np.int32)
    return perm, np.array([n8, n6, K - n8 - n6], dtype=np.int64)


@pytest.mark.parametrize("seed,rows,K", [(0, 3, 70), (1, 5, 32), (2, 2, 129), (3, 4, 7)])
def test_quantize_rows_matches_blockwise_brute_force(seed, rows, K):
    rng = np.random.default_rng(seed)
    src = (rng.normal(0, 1, (rows, K)) * (1 + 30 * (rng.random(K) < 0.1))).astype(np.float32)
    perm, counts = _layout(rng, K)
    codes, scales = oracle.quantize_rows(src, perm, counts)
    offs = np.concatenate([[0], np.cumsum(counts)])
    bits = (8, 6, 4)
    for r in range(rows):
        for g in range(3):
            kr = int(counts[g])
            kp = oracle.pad32(kr)
            vals = [float(src[r, perm[offs[g] + p]]) if p < kr else 0.0 for p in range(kp)]
            for b in range(kp // 32):
                q, e = brute.brute_block(vals[32 * b:32 * b + 32], bits[g])
                assert scales[g][r, b] == e + 127
                nbytes = 32 * bits[g] // 8
                assert bytes(codes[g][r, b * nbytes:(b + 1) * nbytes]) == brute.pack_bits(q, bits[g])


def test_dequantize_rows_matches_python_decode():
    rng = np.random.default_rng(4)
    src = rng.normal(0, 1, (3, 100)).astype(np.float32)
    perm, counts = _layout(rng, 100)
    codes, scales = oracle.quantize_rows(src, perm, counts)
    ref = brute.to_f64(brute.decode_rows(codes, scales, counts))
    assert np.array_equal(oracle.dequantize_rows(codes, scales, counts), ref)


def test_identity_layout_kv():
    rng = np.random.default_rng(5)
    src = rng.normal(0, 1, (4, 128)).astype(np.float32)
    codes, scales = oracle.quantize_rows(src, None, [0, 0, 128])
    assert codes[2].shape == (4, 64) and scales[2].shape == (4, 4)
    for r in range(4):
        for b in range(4):
            q, e = brute.brute_block(src[r, 32 * b:32 * b + 32], 4)
            assert scales[2][r, b] == e + 127
            assert bytes(codes[2][r, 16 * b:16 * b + 16]) == brute.pack_bits(q, 4)


def test_pad_positions_decode_to_zero():
    src = np.ones((2, 33), np.float32)
    codes, scales = oracle.quantize_rows(src, np.arange(33, dtype=np.int32), [0, 0, 33])
    deq = oracle.dequantize_rows(codes, scales, [0, 0, 33])
    assert deq.shape == (2, 64)
    assert np.all(deq[:, :33] == 1.0) and np.all(deq[:, 33:] == 0.0)
    assert np.all(scales[2][:, 1] == 127)     # block 1 holds one real 1.0


@pytest.mark.parametrize("seed,M,N,K", [(0, 5, 7, 70), (1, 3, 4, 200), (2, 1, 9, 33)])
def test_gemm_matches_numpy_of_python_decode(seed, M, N, K):
    rng = np.random.default_rng(seed)
    A = rng.normal(0, 1, (M, K)).astype(np.float32)
    W = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    perm, counts = _layout(rng, K)
    ac, as_ = oracle.quantize_rows(A, perm, counts)
    wc, ws = oracle.quantize_rows(W, perm, counts)
    Y = oracle.gemm(ac, as_, wc, ws, counts)
    da = brute.to_f64(brute.decode_rows(ac, as_, counts))
    dw = brute.to_f64(brute.decode_rows(wc, ws, counts))
    ref = da @ dw.T
    assert Y.shape == (M, N)
    assert np.allclose(Y, ref, rtol=1e-13, atol=1e-13 * np.abs(ref).max())
    # sampled rows / columns return the same entries
    rows, cols = [M - 1, 0], [N - 1, N // 2]
    Ys = oracle.gemm(ac, as_, wc, ws, counts, rows=rows, cols=cols)
    assert np.array_equal(Ys, Y[np.ix_(rows, cols)])


def test_gemm_selector_weights_pick_columns():
    # W row n has a single 1.0 at original column c_n (exact at every width):
    # Y[:, n] must equal the decoded A value of column c_n.
    rng = np.random.default_rng(6)
    K, M = 96, 4
    A = rng.normal(0, 1, (M, K)).astype(np.float32)
    sel = [3, 50, 95, 0]
    W = np.zeros((len(sel), K), np.float32)
    for n, c in enumerate(sel):
        W[n, c] = 1.0
    perm, counts = _layout(rng, K)
    ac, as_ = oracle.quantize_rows(A, perm, counts)
    wc, ws = oracle.quantize_rows(W, perm, counts)
    Y = oracle.gemm(ac, as_, wc, ws, counts)
    deq = oracle.dequantize_rows(ac, as_, counts)
    pos = np.argsort(perm)                     # original column -> real position
    offs = np.concatenate([[0], np.cumsum(counts)])
    pads = np.cumsum([0] + [oracle.pad32(int(c)) for c in counts])
    for n, c in enumerate(sel):
        p = pos[c]
        g = int(np.searchsorted(offs, p, side="right") - 1)
        kpos = pads[g] + (p - offs[g])
        assert np.array_equal(Y[:, n], deq[:, kpos])


def test_all_4bit_layout_equals_plain_blockwise_product():
    rng = np.random.default_rng(7)
    A = rng.normal(0, 1, (3, 64)).astype(np.float32)
    W = rng.normal(0, 1, (5, 64)).astype(np.float32)
    ac, as_ = oracle.quantize_rows(A, None, [0, 0, 64])
    wc, ws = oracle.quantize_rows(W, None, [0, 0, 64])
    Y = oracle.gemm(ac, as_, wc, ws, [0, 0, 64])

    def deq(X):
        out = np.zeros_like(X, dtype=np.float64)
        for r in range(X.shape[0]):
            for b in range(2):
                q, e = brute.brute_block(X[r, 32 * b:32 * b + 32], 4)
                out[r, 32 * b:32 * b + 32] = [float(brute.code_value(c, e, 4)) for c in q]
        return out
    assert np.allclose(Y, deq(A) @ deq(W).T, rtol=1e-14, atol=1e-14)


def test_bf16_tolerance_metric():
    # The bf16 half-ulp used by the GEMM check: 257 rounds to 256 (tie to
    # even) -- a 1/257 relative error that is all output rounding.
    from tests import parity
    import torch
    x = np.array([257.0, 1.0, 3.0, -1000.5, 1e-30])
    hu = parity.half_ulp_bf16(x)
    rounded = torch.tensor(x).to(torch.bfloat16).double().numpy()
    assert np.all(np.abs(rounded - x) <= hu)
    assert parity.gemm_rel_error(np.array([256.0]), np.array([257.0])) == 0.0
    assert parity.gemm_rel_error(np.array([254.0]), np.array([257.0])) > 0.0
    # normwise: one element off by 1 against a max of 4 -> 1/4; rounding of
    # the exact result alone stays within the normwise budget
    assert parity.gemm_normwise_error(np.array([1.0, 4.0]), np.array([2.0, -4.0])) == 2.0
    assert parity.gemm_normwise_error(np.array([1.0, 3.0]), np.array([2.0, 4.0])) == 0.25
    assert parity.gemm_normwise_error(rounded, x) <= parity.GEMM_NORMWISE_TOL
    assert parity.gemm_normwise_error(np.zeros(3), np.zeros(3)) == 0.0
