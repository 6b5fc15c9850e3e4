"""Host-only checks of the C ABI: the library loads, exports every entry point
declared in include/mxs.h, and rejects bad arguments before any launch.
No call here touches a GPU.  The argument checks pass made-up device
addresses, which the library must reject on the host; they run only where no
CUDA device exists, so that a check that stopped rejecting could never reach
a launch on a real GPU (tests/test_gpu_argchecks.py repeats the checks that
can be made with real buffers)."""
import ctypes
import os
import re

import pytest
import torch

fake_pointers = pytest.mark.skipif(torch.cuda.is_available(),
                                   reason="passes made-up device addresses: CPU hosts only")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mxs.h")


@pytest.fixture(scope="module")
def capi():
    from mx_microscaling_mixed_b200 import build
    build.build()
    from mx_microscaling_mixed_b200 import capi as c
    return c


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mxs_[a-z0-9_]+)\s*\(", src)))


def test_header_symbols_exported(capi):
    names = _declared()
    assert len(names) >= 14
    lib = ctypes.CDLL(capi._LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(capi.EXPORTS)


def test_status_strings(capi):
    for st in range(10):
        assert capi.mxs_status_str(st).startswith(capi.STATUS[st])


def test_layout_make_and_sizes(capi):
    lay = capi.mxs_layout_make(256, (13, 38, 205))
    segs = [(s.bits, s.k_real, s.k_pad, s.k_off) for s in lay.c.seg]
    assert segs == [(8, 13, 32, 0), (6, 38, 64, 32), (4, 205, 224, 96)]
    assert lay.K_pad == 320
    cp, cb, sp, sb = capi.mxs_mxtensor_bytes(256, lay)
    assert cp == [32, 48, 112] and cb == [256 * 32, 256 * 48, 256 * 112]
    assert sp == [16, 16, 16] and sb == [256 * 16] * 3
    kv = capi.mxs_layout_make(128, (0, 0, 128))
    cp, cb, sp, sb = capi.mxs_mxtensor_bytes(65536, kv)
    assert cp == [0, 0, 64] and sp == [0, 0, 16]


def test_layout_rejects_bad_counts(capi):
    with pytest.raises(capi.MxsError) as e:
        capi.mxs_layout_make(10, (3, 3, 3))
    assert e.value.status == 2
    with pytest.raises(capi.MxsError):
        capi.mxs_layout_make(10, (-1, 5, 6))


def test_workspace_queries(capi):
    need = ctypes.c_size_t(0)
    assert capi._lib.mxs_sensitivity_workspace_bytes(2048, 4096, 4096, ctypes.byref(need)) == 0
    assert need.value == (32 + 64) * 4096 * 8
    K = (ctypes.c_int64 * 1)(4096)
    assert capi._lib.mxs_allocate_workspace_bytes(1, K, ctypes.byref(need)) == 0
    assert need.value > 2 * 4096 * 4
    assert capi._lib.mxs_sensitivity_workspace_bytes(0, 1, 1, ctypes.byref(need)) == 1


def _fake_tensor(capi, rows, lay, base=1 << 20):
    t = capi.MXTensorC()
    t.rows = rows
    t.lay = lay.c
    cp, cb, sp, sb = capi.mxs_mxtensor_bytes(rows, lay)
    for g in range(3):
        t.codes[g] = base + 4096 * g if cb[g] else None
        t.scales[g] = base + 65536 + 4096 * g if sb[g] else None
        t.code_pitch[g] = cp[g]
        t.scale_pitch[g] = sp[g]
    return t


@fake_pointers
def test_gemm_argument_checks(capi):
    lay = capi.mxs_layout_make(256, (32, 64, 160))
    A = _fake_tensor(capi, 100, lay)
    W = _fake_tensor(capi, 300, lay)
    need = ctypes.c_size_t(0)
    assert capi._lib.mxs_gemm_workspace_bytes(ctypes.byref(A), ctypes.byref(W), ctypes.byref(need)) == 0
    assert need.value >= 100 * 96 * 2 + 300 * 96 * 2 + 100 * 160 + 300 * 160
    # up to 16 activation rows: the decode path stages in shared memory, no workspace
    A8 = _fake_tensor(capi, 8, lay)
    assert capi._lib.mxs_gemm_workspace_bytes(ctypes.byref(A8), ctypes.byref(W), ctypes.byref(need)) == 0
    assert need.value == 0
    # different layouts -> MXS_ERR_SHAPE, no launch
    lay2 = capi.mxs_layout_make(256, (32, 32, 192))
    W2 = _fake_tensor(capi, 300, lay2)
    assert capi._lib.mxs_gemm(ctypes.byref(A), ctypes.byref(W2), 1 << 24, 300, 1 << 26, 1 << 30, None) == 2
    # misaligned code pointer -> MXS_ERR_ALIGN
    A.codes[2] = (1 << 20) + 8
    assert capi._lib.mxs_gemm(ctypes.byref(A), ctypes.byref(W), 1 << 24, 300, 1 << 26, 1 << 30, None) == 3
    # ldy < N -> MXS_ERR_SHAPE
    A.codes[2] = 1 << 21
    assert capi._lib.mxs_gemm(ctypes.byref(A), ctypes.byref(W), 1 << 24, 299, 1 << 26, 1 << 30, None) == 2


@fake_pointers
def test_quantize_argument_checks(capi):
    lay = capi.mxs_layout_make(64, (0, 0, 64))
    t = _fake_tensor(capi, 8, lay)
    # rows mismatch
    assert capi._lib.mxs_quantize_act(1 << 20, 1, 9, 64, ctypes.byref(t), None) == 2
    # bad dtype
    assert capi._lib.mxs_quantize_act(1 << 20, 7, 8, 64, ctypes.byref(t), None) == 4
    # ld < K
    assert capi._lib.mxs_quantize_weight(1 << 20, 0, 8, 32, ctypes.byref(t), None) == 2


@fake_pointers
def test_sensitivity_argument_checks(capi):
    f = capi._lib.mxs_sensitivity
    X, W, H, E, S = 1 << 20, 1 << 24, 1 << 26, 1 << 27, 1 << 28
    need = ctypes.c_size_t(0)
    assert capi._lib.mxs_sensitivity_workspace_bytes(128, 256, 512, ctypes.byref(need)) == 0
    ws, big = 1 << 30, need.value
    # NULL input -> MXS_ERR_ARG
    assert f(None, 1, 128, 512, 512, W, 1, 256, 512, H, E, S, ws, big, None) == 1
    # T < 1 -> MXS_ERR_ARG
    assert f(X, 1, 0, 512, 512, W, 1, 256, 512, H, E, S, ws, big, None) == 1
    # unknown dtype -> MXS_ERR_DTYPE
    assert f(X, 9, 128, 512, 512, W, 1, 256, 512, H, E, S, ws, big, None) == 4
    # pitch below K -> MXS_ERR_SHAPE
    assert f(X, 1, 128, 512, 511, W, 1, 256, 512, H, E, S, ws, big, None) == 2
    assert f(X, 1, 128, 512, 512, W, 1, 256, 500, H, E, S, ws, big, None) == 2
    # more 64-row chunks than one launch takes -> MXS_ERR_SHAPE
    assert f(X, 1, 64 * 65536, 512, 512, W, 1, 256, 512, H, E, S, ws, 1 << 62, None) == 2
    # workspace missing, misaligned or short -> MXS_ERR_WORKSPACE
    assert f(X, 1, 128, 512, 512, W, 1, 256, 512, H, E, S, None, big, None) == 9
    assert f(X, 1, 128, 512, 512, W, 1, 256, 512, H, E, S, ws + 64, big, None) == 9
    assert f(X, 1, 128, 512, 512, W, 1, 256, 512, H, E, S, ws, big - 8, None) == 9


@fake_pointers
def test_gemm_empty_product_needs_no_device(capi):
    lay = capi.mxs_layout_make(256, (32, 64, 160))
    A0 = _fake_tensor(capi, 0, lay)
    W = _fake_tensor(capi, 300, lay)
    # M = 0: nothing to compute, MXS_OK before any device work
    assert capi._lib.mxs_gemm(ctypes.byref(A0), ctypes.byref(W), 1 << 24, 300, None, 0, None) == 0


def _alloc_call(capi, K, N, budget, ws=1 << 30, ws_bytes=1 << 40):
    n = len(K)
    Ks, Ns = (ctypes.c_int64 * n)(*K), (ctypes.c_int64 * n)(*N)
    s = (ctypes.c_void_p * n)(*[(1 << 20) + 65536 * i for i in range(n)])
    perm = (ctypes.c_void_p * n)(*[(1 << 24) + 65536 * i for i in range(n)])
    counts = (ctypes.c_int64 * (3 * n))()
    return capi._lib.mxs_allocate(n, Ks, Ns, s, None, ctypes.byref(budget), perm, counts, ws, ws_bytes, None)


@fake_pointers
def test_allocate_argument_and_budget_checks(capi):
    # budget mode: 4.0 bits on average cannot carry the fixed 32-column 8-bit
    # block -> MXS_ERR_BUDGET, decided on the host before any launch
    b = capi.BudgetC(mode=1, num=4, den=1, fixed8=32)
    assert _alloc_call(capi, [4096], [4096], b) == 5
    assert _alloc_call(capi, [4096, 14336], [4096, 4096], b) == 5
    # a bad mode or denominator -> MXS_ERR_ARG
    assert _alloc_call(capi, [4096], [4096], capi.BudgetC(mode=7, num=9, den=2, fixed8=32)) == 1
    assert _alloc_call(capi, [4096], [4096], capi.BudgetC(mode=1, num=9, den=0, fixed8=32)) == 1
    assert _alloc_call(capi, [4096], [4096], capi.BudgetC(mode=0, p8_num=1, p8_den=0, p6_num=0, p6_den=1)) == 1
    # K < 1 -> MXS_ERR_ARG
    assert _alloc_call(capi, [0], [4096], capi.BudgetC(mode=1, num=9, den=2, fixed8=32)) == 1
    # feasible budget, workspace missing or short -> MXS_ERR_WORKSPACE
    ok = capi.BudgetC(mode=1, num=9, den=2, fixed8=32)
    assert _alloc_call(capi, [4096], [4096], ok, ws=None) == 9
    assert _alloc_call(capi, [4096], [4096], ok, ws_bytes=16) == 9


@fake_pointers
def test_host_checks_survive_random_arguments(capi):
    """Random shapes, pitches and pointers return a status and never crash the
    process.  Some combinations pass every host check and would reach a
    launch on fake pointers, so this runs only where no CUDA device exists
    (the device check then fails first)."""
    import random
    rng = random.Random(1234)
    valid = set(range(10))
    for _ in range(400):
        K = rng.choice([0, 1, 31, 32, 33, 256, 4096, 1 << 20])
        counts = [rng.choice([0, 1, 32, 64, K]) for _ in range(2)]
        counts.append(K - sum(counts))
        try:
            lay = capi.mxs_layout_make(K, counts)
        except Exception:
            continue
        for rows in (0, 1, 16, 2048):
            t = _fake_tensor(capi, rows, lay, base=rng.choice([1 << 20, (1 << 20) + 8]))
            if rng.random() < 0.3:
                t.code_pitch[rng.randrange(3)] = rng.choice([1, 15, 17, 1 << 40])
            w = _fake_tensor(capi, rng.choice([1, 300, 4096]), lay)
            need = ctypes.c_size_t(0)
            assert capi._lib.mxs_gemm_workspace_bytes(ctypes.byref(t), ctypes.byref(w), ctypes.byref(need)) in valid
            assert capi._lib.mxs_gemm(ctypes.byref(t), ctypes.byref(w), rng.choice([None, 1 << 24]),
                                      rng.choice([0, 1, 4096]), rng.choice([None, 1 << 30, (1 << 30) + 4]),
                                      rng.choice([0, 1 << 40]), None) in valid
            dt = rng.choice([0, 1, 2, -1])
            ld = rng.choice([0, K, K + 1, 1 << 33])
            assert capi._lib.mxs_quantize_act(rng.choice([None, 1 << 20, (1 << 20) + 2]), dt, rows, ld,
                                              ctypes.byref(t), None) in valid
            assert capi._lib.mxs_quantize_weight(1 << 20, dt, rows, ld, ctypes.byref(t), None) in valid


@fake_pointers
def test_noalloc_argument_checks(capi):
    """mxs_sensitivity_noalloc returns the codes of mxs_sensitivity and rejects
    shapes beyond its fixed scratch, all before touching the device."""
    f = capi._lib.mxs_sensitivity_noalloc
    X, W, H, E, S = 1 << 20, 1 << 24, 1 << 26, 1 << 27, 1 << 28
    assert f(None, 1, 128, 512, 512, W, 1, 256, 512, H, E, S, None) == 1
    assert f(X, 1, 128, 512, 512, W, 1, 256, 512, None, E, S, None) == 1
    assert f(X, 9, 128, 512, 512, W, 1, 256, 512, H, E, S, None) == 4
    assert f(X, 1, 128, 512, 511, W, 1, 256, 512, H, E, S, None) == 2
    # (ceil(T/64) + ceil(N/64)) * K * 8 bytes > 16 MiB -> MXS_ERR_WORKSPACE
    T, N, K = 64, 64 * 1024, 4096
    assert capi.mxs_sensitivity_workspace_bytes(T, N, K) > capi.NOALLOC_SCRATCH_BYTES
    launches = capi.mxs_launch_count()
    assert f(X, 1, T, K, K, W, 1, N, K, H, E, S, None) == 9
    # the Llama-2-70B MLP shapes exceed it too; the Llama-3-8B down projection fits
    assert capi.mxs_sensitivity_workspace_bytes(2048, 28672, 8192) > capi.NOALLOC_SCRATCH_BYTES
    assert capi.mxs_sensitivity_workspace_bytes(2048, 4096, 14336) <= capi.NOALLOC_SCRATCH_BYTES
    assert capi.mxs_launch_count() == launches
