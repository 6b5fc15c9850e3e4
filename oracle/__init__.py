"""CPU oracle for the MXSens hot path (ctypes wrapper around mxs_oracle.c).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the cpu_baseline / reference leg of ``bench.py`` may import this package.  The
product path (``mx_microscaling_mixed_b200``) never imports it and shares no
code with it; the two meet only in the seeded input generators, which hold
none of the method's arithmetic.

Each function here only marshals numpy arrays; the arithmetic is in
``mxs_oracle.c`` (plain single-threaded C, fp64, no contraction), whose
comments cite the MXSens pages for every step.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mxs_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "liboracle.so")
_lib = None

SEG_BITS = (8, 6, 4)  # segment order of the mixed-width layout
BLOCK = 32


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2 -ffp-contract=off) into oracle/_build."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
            "-fPIC", "-shared", "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32


def _declare(L):
    L.orc_block_exp.argtypes = [_P, ctypes.c_int]
    L.orc_block_exp.restype = ctypes.c_int
    L.orc_quant_block.argtypes = [_P, ctypes.c_int, ctypes.c_int, _P, _P]
    L.orc_quant_block.restype = None
    L.orc_dequant.argtypes = [_I32, ctypes.c_int, ctypes.c_int]
    L.orc_dequant.restype = ctypes.c_double
    L.orc_pack.argtypes = [_P, _I64, ctypes.c_int, _P]
    L.orc_pack.restype = None
    L.orc_unpack.argtypes = [_P, _I64, ctypes.c_int, _P]
    L.orc_unpack.restype = None
    L.orc_sensitivity.argtypes = [_P, _I64, _I64, _P, _I64, _P, _P, _P]
    L.orc_sensitivity.restype = None
    L.orc_rank_order.argtypes = [_P, _I64, _P]
    L.orc_rank_order.restype = None
    L.orc_allocate.argtypes = [ctypes.c_int, _P, _P, _P, _P, ctypes.c_int, _I64, _I64,
                               _I64, _I64, _I64, _I64, _I64, _P, _P]
    L.orc_allocate.restype = ctypes.c_int
    L.orc_quantize_rows.argtypes = [_P, _I64, _I64, _P, _P, _P, _P]
    L.orc_quantize_rows.restype = None
    L.orc_dequantize_rows.argtypes = [_I64, _P, _P, _P, _P]
    L.orc_dequantize_rows.restype = None
    L.orc_gemm.argtypes = [_I64, _I64, _P, _P, _P, _P, _P, _P, _I64, _P, _I64, _P]
    L.orc_gemm.restype = None
    L.orc_attn_decode.argtypes = [_P, _I64, _I64, _P, _P, _P, _P, _I64, _I64, ctypes.c_double, _P]
    L.orc_attn_decode.restype = None


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _f64(x) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    if not np.all(np.isfinite(a)):
        raise ValueError("oracle inputs must be finite")
    return a


def pad32(n: int) -> int:
    return (n + BLOCK - 1) // BLOCK * BLOCK


# ---------------------------------------------------------------- C1 format
def block_exp(x) -> int:
    x = _f64(x)
    return lib().orc_block_exp(_ptr(x), x.size)


def quant_block(x, m: int):
    """Codes (int32) and shared exponent of one block at width m."""
    x = _f64(x)
    q = np.zeros(x.size, dtype=np.int32)
    e = ctypes.c_int(0)
    lib().orc_quant_block(_ptr(x), x.size, m, _ptr(q), ctypes.byref(e))
    return q, e.value


def dequant(q, e: int, m: int) -> np.ndarray:
    return np.array([lib().orc_dequant(int(v), e, m) for v in np.asarray(q).ravel()])


def pack(q, m: int) -> np.ndarray:
    q = np.ascontiguousarray(np.asarray(q, dtype=np.int32))
    out = np.zeros(q.size * m // 8, dtype=np.uint8)
    lib().orc_pack(_ptr(q), q.size, m, _ptr(out))
    return out


def unpack(b, n: int, m: int) -> np.ndarray:
    b = np.ascontiguousarray(np.asarray(b, dtype=np.uint8))
    q = np.zeros(n, dtype=np.int32)
    lib().orc_unpack(_ptr(b), n, m, _ptr(q))
    return q


# ---------------------------------------------------------- C2 sensitivity
def sensitivity(X, W):
    """(H_diag, E, s) for calibration X (T x K) and weight W (N x K)."""
    X = _f64(X)
    W = _f64(W)
    T, K = X.shape
    N, K2 = W.shape
    assert K == K2
    H = np.zeros(K)
    E = np.zeros(K)
    s = np.zeros(K)
    lib().orc_sensitivity(_ptr(X), T, K, _ptr(W), N, _ptr(H), _ptr(E), _ptr(s))
    return H, E, s


# ------------------------------------------------------------ C3 allocation
def rank_order(s) -> np.ndarray:
    s = _f64(s)
    order = np.zeros(s.size, dtype=np.int32)
    lib().orc_rank_order(_ptr(s), s.size, _ptr(order))
    return order


def allocate(s_list, N_list, *, mode: str, budget=(9, 2), p8=(5, 100), p6=(15, 100),
             fixed8: int = 32, layer_w=None):
    """Bit allocation over layers.  mode 'fractions', 'budget' or 'layer'
    (the layer-score rule; layer_w holds the layer scores).

    Returns (perms, counts) with counts an (L, 3) int64 array of (n8, n6, n4).
    Raises ValueError if the fixed 8-bit blocks exceed the budget."""
    s_arrs = [_f64(s) for s in s_list]
    Lc = len(s_arrs)
    K = np.array([a.size for a in s_arrs], dtype=np.int64)
    N = np.array(N_list, dtype=np.int64)
    sp = (ctypes.c_void_p * Lc)(*[a.ctypes.data for a in s_arrs])
    perms = [np.zeros(max(int(k), 1), dtype=np.int32) for k in K]
    pp = (ctypes.c_void_p * Lc)(*[p.ctypes.data for p in perms])
    counts = np.zeros((Lc, 3), dtype=np.int64)
    w = None if layer_w is None else _f64(layer_w)
    rc = lib().orc_allocate(Lc, _ptr(K), _ptr(N), ctypes.cast(sp, ctypes.c_void_p),
                            None if w is None else _ptr(w),
                            {"fractions": 0, "budget": 1, "layer": 2}[mode],
                            int(budget[0]), int(budget[1]), int(p8[0]), int(p8[1]),
                            int(p6[0]), int(p6[1]), int(fixed8),
                            ctypes.cast(pp, ctypes.c_void_p), _ptr(counts))
    if rc == 1:
        raise ValueError("budget infeasible: fixed 8-bit blocks exceed it")
    if rc != 0:
        raise ValueError("bad allocation arguments")
    return [p[:int(k)] for p, k in zip(perms, K)], counts


# ----------------------------------------------------------- C4 quantizers
def segment_row_bytes(counts):
    return [pad32(int(c)) * b // 8 for c, b in zip(counts, SEG_BITS)]


def segment_scale_cols(counts):
    return [pad32(int(c)) // BLOCK for c in counts]


def quantize_rows(src, perm, counts):
    """Compact codes and scales, one (rows x bytes) uint8 array per segment."""
    src = _f64(src)
    rows, K = src.shape
    counts = np.ascontiguousarray(np.asarray(counts, dtype=np.int64))
    assert int(counts.sum()) == K
    rb = segment_row_bytes(counts)
    sb = segment_scale_cols(counts)
    codes = [np.zeros((rows, max(b, 0)), dtype=np.uint8) for b in rb]
    scales = [np.zeros((rows, max(b, 0)), dtype=np.uint8) for b in sb]
    cp = (ctypes.c_void_p * 3)(*[c.ctypes.data for c in codes])
    sp = (ctypes.c_void_p * 3)(*[s.ctypes.data for s in scales])
    pr = None
    if perm is not None:
        perm = np.ascontiguousarray(np.asarray(perm, dtype=np.int32))
        pr = _ptr(perm)
    lib().orc_quantize_rows(_ptr(src), rows, K, pr, _ptr(counts),
                            ctypes.cast(cp, ctypes.c_void_p), ctypes.cast(sp, ctypes.c_void_p))
    return codes, scales


def dequantize_rows(codes, scales, counts) -> np.ndarray:
    counts = np.ascontiguousarray(np.asarray(counts, dtype=np.int64))
    rows = next((c.shape[0] for c in codes if c.size), 0)
    if rows == 0:
        rows = max(c.shape[0] for c in codes)
    kp = sum(pad32(int(c)) for c in counts)
    out = np.zeros((rows, kp))
    codes = [np.ascontiguousarray(c) for c in codes]
    scales = [np.ascontiguousarray(s) for s in scales]
    cp = (ctypes.c_void_p * 3)(*[c.ctypes.data for c in codes])
    sp = (ctypes.c_void_p * 3)(*[s.ctypes.data for s in scales])
    lib().orc_dequantize_rows(rows, _ptr(counts), ctypes.cast(cp, ctypes.c_void_p),
                              ctypes.cast(sp, ctypes.c_void_p), _ptr(out))
    return out


# ---------------------------------------------------------------- C5 GEMM
def gemm(a_codes, a_scales, w_codes, w_scales, counts, rows=None, cols=None):
    """fp64 Y[rows, cols] of the mixed-width product (all rows/cols if None)."""
    counts = np.ascontiguousarray(np.asarray(counts, dtype=np.int64))
    M = max(c.shape[0] for c in a_codes)
    N = max(c.shape[0] for c in w_codes)
    rows = np.arange(M, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    cols = np.arange(N, dtype=np.int64) if cols is None else np.asarray(cols, dtype=np.int64)
    rows = np.ascontiguousarray(rows)
    cols = np.ascontiguousarray(cols)
    assert rows.size == 0 or (rows.min() >= 0 and rows.max() < M)
    assert cols.size == 0 or (cols.min() >= 0 and cols.max() < N)
    Y = np.zeros((rows.size, cols.size))
    arrs = [np.ascontiguousarray(x) for x in (*a_codes, *a_scales, *w_codes, *w_scales)]
    ptrs = [(ctypes.c_void_p * 3)(*[a.ctypes.data for a in arrs[3 * i:3 * i + 3]])
            for i in range(4)]
    lib().orc_gemm(M, N, _ptr(counts), *[ctypes.cast(p, ctypes.c_void_p) for p in ptrs],
                   _ptr(rows), rows.size, _ptr(cols), cols.size, _ptr(Y))
    return Y


# ------------------------------------------------- decode attention (KV4)
def attn_decode(q, k_codes, k_scales, v_codes, v_scales, T: int, n_kvh: int, sm_scale: float) -> np.ndarray:
    """fp64 output (n_qh x d) of one decode step of grouped-query attention
    over MXINT4 K/V caches given as compact codes (T*n_kvh x d/2 bytes) and
    scales (T*n_kvh x d/32 bytes), rows token-major."""
    q = _f64(q)
    n_qh, d = q.shape
    assert d % BLOCK == 0 and n_qh % n_kvh == 0
    arrs = [np.ascontiguousarray(np.asarray(a, dtype=np.uint8)) for a in (k_codes, k_scales, v_codes, v_scales)]
    for a, w in zip(arrs, (d // 2, d // BLOCK, d // 2, d // BLOCK)):
        assert a.shape == (T * n_kvh, w), (a.shape, T, n_kvh, w)
    out = np.zeros((n_qh, d))
    lib().orc_attn_decode(_ptr(q), n_qh, d, *[_ptr(a) for a in arrs], int(T), int(n_kvh), float(sm_scale),
                          _ptr(out))
    return out
