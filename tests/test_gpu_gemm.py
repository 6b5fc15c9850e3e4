"""GPU parity: mxs_gemm against the oracle's fp64 product of the dequantised
operands, max relative error <= 2e-3 (denominator floored at 1% of max|Y|).
Both sides quantise the same device bytes with the same layout; the oracle
quantises independently (its codes are checked equal to the GPU's in
test_gpu_quantize)."""
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


def _layout(c, K, counts, seed):
    perm = np.random.default_rng(seed).permutation(K).astype(np.int32)
    return c.mxs_layout_make(K, counts, torch.from_numpy(perm).cuda()), perm


def _run(c, A, W, counts, seed=0, rows=None, cols=None):
    K = A.shape[1]
    lay, perm = _layout(c, K, counts, seed)
    Aq = c.mxtensor_empty(A.shape[0], lay)
    Wq = c.mxtensor_empty(W.shape[0], lay)
    c.mxs_quantize_act(A, Aq)
    c.mxs_quantize_weight(W, Wq)
    Y = c.mxs_gemm(Aq, Wq)
    c.mxs_sync()
    ac, as_ = oracle.quantize_rows(parity.host64(A), perm, counts)
    wc, ws = oracle.quantize_rows(parity.host64(W), perm, counts)
    Yref = oracle.gemm(ac, as_, wc, ws, counts, rows=rows, cols=cols)
    Yg = Y.float().cpu().numpy().astype(np.float64)
    if rows is not None or cols is not None:
        r = np.arange(A.shape[0]) if rows is None else np.asarray(rows)
        cc = np.arange(W.shape[0]) if cols is None else np.asarray(cols)
        Yg = Yg[np.ix_(r, cc)]
    return Yg, Yref


SHAPES = [
    # M, N, K, counts
    (128, 256, 256, (13, 38, 205)),
    (1, 8, 32, (0, 0, 32)),
    (200, 300, 270, (40, 70, 160)),
    (128, 256, 256, (256, 0, 0)),
    (130, 260, 96, (0, 96, 0)),
    (257, 513, 640, (32, 96, 512)),
    (64, 1000, 1000, (32, 200, 768)),
    (300, 200, 33, (1, 0, 32)),
    (16, 256, 4096, (32, 960, 3104)),
]


@pytest.mark.parametrize("M,N,K,counts", SHAPES)
def test_gemm_matches_oracle(c, M, N, K, counts):
    A = inputs.random_matrix(M, K, device="cuda", seed=M + K, dtype=torch.bfloat16)
    W = inputs.random_matrix(N, K, device="cuda", seed=N + 2 * K, dtype=torch.bfloat16, std=0.02)
    Y, Yref = _run(c, A, W, counts, seed=K)
    err, nw = parity.gemm_rel_error(Y, Yref), parity.gemm_normwise_error(Y, Yref)
    print(f"M={M} N={N} K={K}: max rel err {err:.3e}, normwise {nw:.3e}")
    assert err <= parity.GEMM_TOL, f"max rel err {err:.3e}"
    assert nw <= parity.GEMM_NORMWISE_TOL, f"normwise {nw:.3e}"


def test_parity_layer_fp32_inputs(c):
    d = inputs.parity_layer("cuda", seed=0)
    Y, Yref = _run(c, d["A"], d["W"], (13, 38, 205), seed=1)
    assert parity.gemm_rel_error(Y, Yref) <= parity.GEMM_TOL


def test_full_attention_prefill_sampled(c):
    A = inputs.gaussian_acts("cuda", seed=2002, rows=2048, K=4096)
    W = inputs.attn_weight("cuda", seed=2000)
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(2048, 48, replace=False))
    rows[-1] = 2047
    cols = np.sort(rng.choice(4096, 64, replace=False))
    cols[0] = 0
    Y, Yref = _run(c, A, W, (32, 960, 3104), seed=7, rows=rows, cols=cols)
    assert parity.gemm_rel_error(Y, Yref) <= parity.GEMM_TOL


@pytest.mark.parametrize("M", [1, 16])
def test_full_attention_decode(c, M):
    A = inputs.gaussian_acts("cuda", seed=2003, rows=M, K=4096)
    W = inputs.attn_weight("cuda", seed=2000)
    cols = np.arange(0, 4096, 37)
    Y, Yref = _run(c, A, W, (32, 960, 3104), seed=8, cols=cols)
    assert parity.gemm_rel_error(Y, Yref) <= parity.GEMM_TOL


def test_selector_weights_are_exact(c):
    # W rows with a single 1.0 select decoded A values: exact in bf16 output
    K, M = 256, 130
    A = inputs.random_matrix(M, K, device="cuda", seed=3, dtype=torch.bfloat16)
    W = torch.zeros(64, K, dtype=torch.bfloat16, device="cuda")
    sel = np.random.default_rng(1).choice(K, 64, replace=False)
    W[np.arange(64), sel] = 1.0
    Y, Yref = _run(c, A, W, (32, 64, 160), seed=2)
    assert np.array_equal(Y, Yref)


def test_selector_extreme_scales_exact(c):
    """Rows of A scaled across the exponent range (block scale bytes from ~10
    to ~252) pass the staging conversions -- including the packed bf16 path
    for 6-bit blocks and its fp32 fallback at the range ends -- exactly."""
    K, M = 256, 24
    A = inputs.random_matrix(M, K, device="cuda", seed=4, dtype=torch.float32, outlier_frac=0.0)
    ks = [-118, -117, -116, -115, -114, -100, -60, -1, 0, 1, 60, 100, 118, 119, 120, 121, 122, 122,
          -113, 30, -30, 90, -90, 2]
    A = (A * torch.tensor([2.0 ** k for k in ks], device="cuda")[:, None]).to(torch.bfloat16)
    W = torch.zeros(64, K, dtype=torch.bfloat16, device="cuda")
    sel = np.random.default_rng(5).choice(K, 64, replace=False)
    W[np.arange(64), sel] = 1.0
    Y, Yref = _run(c, A, W, (32, 64, 160), seed=6)
    assert np.array_equal(Y, Yref)


def test_zero_k_segments_and_strided_output(c):
    K = 128
    A = inputs.random_matrix(70, K, device="cuda", seed=5, dtype=torch.bfloat16)
    W = inputs.random_matrix(90, K, device="cuda", seed=6, dtype=torch.bfloat16)
    lay, perm = _layout(c, K, (0, 0, K), 3)
    Aq, Wq = c.mxtensor_empty(70, lay), c.mxtensor_empty(90, lay)
    c.mxs_quantize_act(A, Aq)
    c.mxs_quantize_weight(W, Wq)
    Ybig = torch.full((70, 104), 7.0, dtype=torch.bfloat16, device="cuda")
    c.mxs_gemm(Aq, Wq, Y=Ybig[:, :90])
    c.mxs_sync()
    assert torch.all(Ybig[:, 90:] == 7.0)
    ac, as_ = oracle.quantize_rows(parity.host64(A), perm, (0, 0, K))
    wc, ws = oracle.quantize_rows(parity.host64(W), perm, (0, 0, K))
    Yref = oracle.gemm(ac, as_, wc, ws, (0, 0, K))
    assert parity.gemm_rel_error(Ybig[:, :90].float().cpu().numpy().astype(np.float64), Yref) <= parity.GEMM_TOL


SMALL_M = [
    # M, N, K, counts -- every activation-row template (1, 2, 4, 8, 16), K chunking
    # (K = 14336 at M = 16 spans several staged chunks), ragged N, and M = 17
    # just past the decode path.
    (2, 100, 200, (32, 64, 104)),
    (3, 37, 96, (0, 32, 64)),
    (5, 260, 512, (32, 96, 384)),
    (8, 130, 1000, (40, 200, 760)),
    (12, 300, 4096, (32, 960, 3104)),      # the attention layer's width, W staged beside A
    (11, 64, 14336, (32, 3520, 10784)),
    (16, 96, 14336, (32, 3520, 10784)),
    # K = 14336 with 9 activation rows over 7 W-row tiles (the last ragged):
    # W streams from global memory beside the staged activations
    (9, 100, 14336, (32, 3520, 10784)),
    (16, 40, 28672, (32, 3520, 25120)),    # the 70B down projection's width
    (17, 300, 640, (32, 96, 512)),
]


@pytest.mark.parametrize("M,N,K,counts", SMALL_M)
def test_gemm_small_m_matches_oracle(c, M, N, K, counts):
    A = inputs.random_matrix(M, K, device="cuda", seed=3 * M + K, dtype=torch.bfloat16)
    W = inputs.random_matrix(N, K, device="cuda", seed=N + K, dtype=torch.bfloat16, std=0.02)
    Y, Yref = _run(c, A, W, counts, seed=M)
    err, nw = parity.gemm_rel_error(Y, Yref), parity.gemm_normwise_error(Y, Yref)
    print(f"M={M} N={N} K={K}: max rel err {err:.3e}, normwise {nw:.3e}")
    assert err <= parity.GEMM_TOL, f"max rel err {err:.3e}"
    assert nw <= parity.GEMM_NORMWISE_TOL, f"normwise {nw:.3e}"


@pytest.mark.parametrize("M", [4, 16])
def test_gemm_small_m_extreme_codes(c, M):
    # blocks at the clamp (all codes +-(2^(m-1)-1)) in every segment, through
    # the GEMV (M = 4) and the integer-MMA kernel (M = 16)
    K = 256
    A = torch.full((M, K), 1.96875, dtype=torch.bfloat16, device="cuda")
    A[:, 1::2] = -1.96875
    W = torch.full((40, K), -1.96875, dtype=torch.bfloat16, device="cuda")
    Y, Yref = _run(c, A, W, (64, 64, 128), seed=9)
    assert parity.gemm_rel_error(Y, Yref) <= parity.GEMM_TOL


PAIR_SHAPES = [
    # M >= 512 runs the 2-CTA pair kernel (256 x 240 tiles, persistent)
    (512, 256, 4096, (32, 960, 3104)),
    (600, 700, 640, (32, 96, 512)),          # ragged M and N tiles
    (512, 512, 256, (256, 0, 0)),            # 8-bit only: bf16 MMAs only
    (520, 300, 320, (0, 0, 320)),            # 4-bit only: block-scaled MMAs only
    (2560, 2048, 256, (32, 64, 160)),        # 80 tiles > 74 pairs: persistent loop
]


@pytest.mark.parametrize("M,N,K,counts", PAIR_SHAPES)
def test_gemm_pair_kernel_matches_oracle(c, M, N, K, counts):
    A = inputs.random_matrix(M, K, device="cuda", seed=M + 5 * K, dtype=torch.bfloat16)
    W = inputs.random_matrix(N, K, device="cuda", seed=N + 7 * K, dtype=torch.bfloat16, std=0.02)
    Y, Yref = _run(c, A, W, counts, seed=M + N)
    err, nw = parity.gemm_rel_error(Y, Yref), parity.gemm_normwise_error(Y, Yref)
    print(f"M={M} N={N} K={K}: max rel err {err:.3e}, normwise {nw:.3e}")
    assert err <= parity.GEMM_TOL, f"max rel err {err:.3e}"
    assert nw <= parity.GEMM_NORMWISE_TOL, f"normwise {nw:.3e}"
