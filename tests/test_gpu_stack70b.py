"""GPU parity on the Llama-2-70B-shaped stack with all 80 layers' weights
quantised in place: 560 matrices (q, o 8192x8192; k, v 1024x8192; gate, up
28672x8192; down 8192x28672), N(0, 0.015^2) with 2% of the columns x20, each
generated on the device in bf16, scored on a 2048-row calibration X of its
input width, allocated at 4.25 bits and quantised into storage that stays
resident (about 38.5 GB of codes and scales) while its bf16 is freed.

Checked: every allocation meets the 4.25-bit budget exactly with the 32
fixed 8-bit columns; after the whole stack is stored (so that no buffer was
overwritten by a later one), sampled rows of sampled matrices carry exactly
the oracle's codes and scales for the bytes the GPU was given (copied back
before the bf16 was freed) under the GPU's allocation; and a decode product
over the last layer's down projection matches the oracle's fp64 product of
the dequantised operands within the GEMM tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
from mx_microscaling_mixed_b200 import inputs
from tests import parity

pytestmark = pytest.mark.gpu

SHAPES = (("q", 8192, 8192), ("k", 1024, 8192), ("v", 1024, 8192), ("o", 8192, 8192),
          ("gate", 28672, 8192), ("up", 28672, 8192), ("down", 8192, 28672))
LAYERS = 80
BUDGET = (17, 4)
CHECK = {(0, 1), (0, 6), (41, 4), (79, 0), (79, 6)}      # (layer, matrix) sampled against the oracle


@pytest.fixture(scope="module")
def c():
    parity.need_gpu()
    return parity.capi()


def test_stack70b_inplace(c):
    X = {K: inputs.gaussian_acts("cuda", 4999 - i, 2048, K) for i, K in enumerate((8192, 28672))}
    store, kept = [], {}
    packed = 0
    for layer in range(LAYERS):
        for j, (_, N, K) in enumerate(SHAPES):
            W = inputs.random_matrix(N, K, device="cuda", seed=5000 + 16 * layer + j, dtype=torch.bfloat16,
                                     std=0.015, outlier_frac=0.02, outlier_scale=20.0)
            _, _, s = c.mxs_sensitivity(X[K], W)
            perms, counts = c.mxs_allocate([s], [N], mode="budget", budget=BUDGET)
            n8, n6, n4 = counts[0]
            assert n8 == 32 and n8 + n6 + n4 == K
            assert 4 * (8 * n8 + 6 * n6 + 4 * n4) == BUDGET[0] * K        # exactly 4.25 bits
            lay = c.mxs_layout_make(K, counts[0], perms[0])
            Wq = c.mxtensor_empty(N, lay)
            c.mxs_quantize_weight(W, Wq)
            if (layer, j) in CHECK:
                rows = np.sort(np.random.default_rng(7 * layer + j).choice(N, 4, replace=False))
                kept[(layer, j)] = (rows, parity.host64(W[torch.from_numpy(rows).cuda()]),
                                    perms[0].cpu().numpy(), tuple(counts[0]))
            packed += sum(t.numel() for t in Wq.codes + Wq.scales if t is not None)
            store.append(Wq)
            del W, s
    c.mxs_sync()
    assert 36e9 < packed < 41e9, packed

    for (layer, j), (rows, src, perm, cnt) in kept.items():
        Wq = store[len(SHAPES) * layer + j]
        oc, os_ = oracle.quantize_rows(src, perm, cnt)
        idx = torch.from_numpy(rows).cuda()
        for g in range(3):
            assert np.array_equal(Wq.code_rows(g)[idx].cpu().numpy(), oc[g]), (layer, j, g)
            assert np.array_equal(Wq.scale_rows(g)[idx].cpu().numpy(), os_[g]), (layer, j, g)

    # decode over the last layer's down projection: the 4 sampled output columns
    rows, src, perm, cnt = kept[(LAYERS - 1, 6)]
    Wq = store[-1]
    A = inputs.gaussian_acts("cuda", 4990, 1, 28672)
    Aq = c.mxtensor_empty(1, Wq.layout)
    c.mxs_quantize_act(A, Aq)
    Y = c.mxs_gemm(Aq, Wq)
    c.mxs_sync()
    ac, as_ = oracle.quantize_rows(parity.host64(A), perm, cnt)
    wc, ws = oracle.quantize_rows(src, perm, cnt)
    Yref = oracle.gemm(ac, as_, wc, ws, cnt)
    Yg = Y[:, torch.from_numpy(rows).cuda()].float().cpu().numpy().astype(np.float64)
    err = parity.gemm_rel_error(Yg, Yref)
    assert err <= parity.GEMM_TOL, f"max rel err {err:.3e}"
