"""GPU parity at the full sizes of the MLP-shaped and 70B-shaped workloads.

The device quantises and multiplies the whole matrices, in the launch
configurations the library picks for those sizes; the oracle, which would
take minutes on the full matrices, quantises only sampled rows (codes and
scales compared byte for byte) and computes only sampled outputs of the
GEMM (within the GEMM tolerance).  Counts follow the workloads' average-bit
budgets with the 32 always-8-bit columns: n6 = (budget - 4) K / 2 - 64.
"""
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


def _counts(K, budget):
    n6 = int(round((budget - 4.0) * K / 2)) - 64
    return (32, n6, K - 32 - n6)


def _sample(n, k, seed):
    rows = np.sort(np.random.default_rng(seed).choice(n, k, replace=False))
    rows[0], rows[-1] = 0, n - 1
    return np.unique(rows)


def _layout(c, K, counts, seed):
    perm = np.random.default_rng(seed).permutation(K).astype(np.int32)
    return c.mxs_layout_make(K, counts, torch.from_numpy(perm).cuda()), perm


def _check_rows(t, src, rows, perm, counts, what):
    """Codes and scales of the sampled rows of GPU tensor t against the oracle."""
    oc, os_ = oracle.quantize_rows(parity.host64(src[torch.from_numpy(rows).cuda()]), perm, counts)
    for g in range(3):
        cg = t.code_rows(g).cpu().numpy()[rows]
        sg = t.scale_rows(g).cpu().numpy()[rows]
        assert np.array_equal(cg, oc[g]), f"{what}: segment {g} codes differ"
        assert np.array_equal(sg, os_[g]), f"{what}: segment {g} scales differ"
    return oc, os_


def _gemm_sampled(c, A, W, counts, seed, rows, cols):
    K = A.shape[1]
    lay, perm = _layout(c, K, counts, seed)
    Aq = c.mxtensor_empty(A.shape[0], lay)
    Wq = c.mxtensor_empty(W.shape[0], lay)
    c.mxs_quantize_act(A, Aq)
    c.mxs_quantize_weight(W, Wq)
    Y = c.mxs_gemm(Aq, Wq)
    c.mxs_sync()
    ac, as_ = _check_rows(Aq, A, rows, perm, counts, "activations")
    wc, ws = _check_rows(Wq, W, cols, perm, counts, "weights")
    Yref = oracle.gemm(ac, as_, wc, ws, counts)
    Yg = Y[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()].float().cpu().numpy().astype(np.float64)
    err, nw = parity.gemm_rel_error(Yg, Yref), parity.gemm_normwise_error(Yg, Yref)
    print(f"sampled {len(rows)} x {len(cols)}: max rel err {err:.3e}, normwise {nw:.3e}")
    assert err <= parity.GEMM_TOL, f"max rel err {err:.3e}"
    assert nw <= parity.GEMM_NORMWISE_TOL, f"normwise {nw:.3e}"


def test_mlp_gate_up_prefill_M8192(c):
    """Gate/up projection W 14336 x 4096 at M = 8192 (2-CTA tcgen05 path)."""
    K = 4096
    A = inputs.gaussian_acts("cuda", seed=5001, rows=8192, K=K)
    W = inputs.attn_weight("cuda", seed=5000, N=14336, K=K)
    _gemm_sampled(c, A, W, _counts(K, 4.5), seed=11, rows=_sample(8192, 40, 1), cols=_sample(14336, 40, 2))


def test_mlp_down_prefill_M8192(c):
    """Down projection W 4096 x 14336 at M = 8192: the longest call of the
    layer step (2-CTA tcgen05 path, K = 14336)."""
    d = inputs.mlp_down_layer("cuda", seed=3000, M=8192)
    _gemm_sampled(c, d["A"], d["W"], _counts(14336, 4.5), seed=12, rows=_sample(8192, 40, 5),
                  cols=_sample(4096, 40, 6))


def test_mlp_down_prefill_M2048(c):
    """Down projection W 4096 x 14336 on SwiGLU-like Laplace inputs with spikes."""
    d = inputs.mlp_down_layer("cuda", seed=3000, M=2048)
    _gemm_sampled(c, d["A"], d["W"], _counts(14336, 4.5), seed=12, rows=_sample(2048, 40, 3),
                  cols=_sample(4096, 40, 4))


@pytest.mark.parametrize("M", [1, 16])
def test_mlp_down_decode(c, M):
    """K = 14336 decode: at M = 16 the W rows do not fit beside the activations
    and stream from global memory."""
    A = inputs.laplace_acts("cuda", seed=3100 + M, rows=M, K=14336)
    W = inputs.attn_weight("cuda", seed=3000, N=4096, K=14336)
    _gemm_sampled(c, A, W, _counts(14336, 4.5), seed=13, rows=np.arange(M), cols=_sample(4096, 96, 5))


def test_70b_up_prefill_M4096(c):
    """70B-shaped W 28672 x 8192 at M = 4096, budget 4.25 bits (rows too wide for
    the transposed quantiser: the staged-row kernel)."""
    K = 8192
    A = inputs.gaussian_acts("cuda", seed=6001, rows=4096, K=K)
    W = inputs.attn_weight("cuda", seed=6000, N=28672, K=K, std=0.015)
    _gemm_sampled(c, A, W, _counts(K, 4.25), seed=14, rows=_sample(4096, 32, 6), cols=_sample(28672, 32, 7))


def test_70b_down_decode_M1(c):
    """70B-shaped W 8192 x 28672 at M = 1."""
    K = 28672
    A = inputs.gaussian_acts("cuda", seed=6101, rows=1, K=K)
    W = inputs.attn_weight("cuda", seed=6100, N=8192, K=K, std=0.015)
    _gemm_sampled(c, A, W, _counts(K, 4.25), seed=15, rows=np.arange(1), cols=_sample(8192, 96, 8))


def test_70b_kv_proj_prefill_M4096(c):
    """70B-shaped k/v projection W 1024 x 8192 at M = 4096 (few output tiles)."""
    K = 8192
    A = inputs.gaussian_acts("cuda", seed=6201, rows=4096, K=K)
    W = inputs.attn_weight("cuda", seed=6200, N=1024, K=K, std=0.015)
    _gemm_sampled(c, A, W, _counts(K, 4.25), seed=16, rows=_sample(4096, 32, 9), cols=_sample(1024, 48, 10))
