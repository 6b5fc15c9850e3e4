"""GPU parity: mxs_attn_decode (one decode step of grouped-query attention
reading the MXINT4 K/V cache) against the fp64 oracle on the same bytes.

The cache is quantised on the GPU (mxs_quantize_act, identity layout), its
code and scale bytes are read back and handed to the oracle together with the
bf16 query.  Error metric per query head: max_d |O - Oref| divided by the
largest decoded value magnitude of that head's V rows (the output is a
convex combination of those rows).  Budget ATTN_TOL, derived from the
kernel's arithmetic: decoded values are exact; scores accumulate 128 exact
products in fp32 (|error| <= 128 * 2^-24 * sum|q k| * sm_scale, about
6e-5 at the workload's scale, which moves a weight by that relative amount);
exp2 is within 2^-22; the weights enter the output product with 16
significant bits (2^-17); the output sums at most 256 tokens per split and
32 splits in fp32 (< 2e-5).  Together below 1.5e-4 of max|V|; the test
allows 5e-4 (1e-3 for the sharpened softmax, whose scores are 4x larger).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from mx_microscaling_mixed_b200 import inputs
from tests import parity

pytestmark = pytest.mark.gpu

ATTN_TOL = 5e-4


@pytest.fixture(scope="module")
def c():
    parity.need_gpu()
    return parity.capi()


def _cache(c, T, n_kvh, seed, scale=1.0):
    kv = inputs.kv_cache("cuda", seed, T, n_kvh, 128).reshape(-1, 128)
    if scale != 1.0:
        kv = (kv.float() * scale).to(torch.bfloat16)
    lay = c.mxs_layout_make(128, (0, 0, 128))
    t = c.mxtensor_empty(kv.shape[0], lay)
    c.mxs_quantize_act(kv, t)
    return t


def _run(c, T, n_qh, n_kvh, seed, sm_scale=None, q_scale=1.0):
    K = _cache(c, T, n_kvh, seed)
    V = _cache(c, T, n_kvh, seed + 1)
    q = (inputs.random_matrix(n_qh, 128, device="cuda", seed=seed + 2, dtype=torch.float32, outlier_frac=0.0)
         * q_scale).to(torch.bfloat16)
    sm = 1.0 / math.sqrt(128) if sm_scale is None else sm_scale
    out = c.mxs_attn_decode(q, K, V, T, n_kvh, sm)
    c.mxs_sync()
    kc, ks = parity.compact(K, 2)
    vc, vs = parity.compact(V, 2)
    ref = oracle.attn_decode(parity.host64(q), kc, ks, vc, vs, T, n_kvh, sm)
    vdec = oracle.dequantize_rows([np.zeros((T * n_kvh, 0), np.uint8)] * 2 + [vc],
                                  [np.zeros((T * n_kvh, 0), np.uint8)] * 2 + [vs], [0, 0, 128])
    got = out.cpu().numpy().astype(np.float64)
    rep = n_qh // n_kvh
    errs = []
    for h in range(n_qh):
        vmax = np.abs(vdec[h // rep::n_kvh]).max()
        errs.append(np.abs(got[h] - ref[h]).max() / vmax)
    norm = np.abs(got - ref).max() / np.abs(ref).max()
    return max(errs), norm


@pytest.mark.parametrize("T,n_qh,n_kvh", [
    (8192, 32, 8),       # the Llama-3-8B cache: 8192 tokens x 8 kv heads, 32 query heads
    (1, 32, 8),          # one token: the output is its value row
    (17, 4, 2),          # one split, a ragged 16-token tile
    (1000, 8, 8),        # one query head per kv head
    (3001, 64, 8),       # eight query heads per kv head (Llama-2-70B grouping), ragged splits
    (300, 16, 2),
])
def test_matches_oracle(c, T, n_qh, n_kvh):
    err, norm = _run(c, T, n_qh, n_kvh, seed=100 + T)
    print(f"T={T} n_qh={n_qh} n_kvh={n_kvh}: max err / max|V| = {err:.2e}, normwise {norm:.2e}")
    assert err <= ATTN_TOL


def test_sharp_softmax(c):
    # scores four times larger: weights concentrate on a few tokens
    err, norm = _run(c, 2048, 32, 8, seed=7, q_scale=4.0)
    print(f"sharp: max err / max|V| = {err:.2e}, normwise {norm:.2e}")
    assert err <= 2 * ATTN_TOL


def test_deterministic_and_argument_checks(c):
    T, n_qh, n_kvh = 512, 32, 8
    K, V = _cache(c, T, n_kvh, 1), _cache(c, T, n_kvh, 2)
    q = inputs.random_matrix(n_qh, 128, device="cuda", seed=3, dtype=torch.bfloat16, outlier_frac=0.0)
    a = c.mxs_attn_decode(q, K, V, T, n_kvh, 0.1)
    b = c.mxs_attn_decode(q, K, V, T, n_kvh, 0.1)
    c.mxs_sync()
    assert torch.equal(a, b)
    n0 = c.mxs_launch_count()
    for args in ((q, K, V, T, 5, 0.1),        # n_qh not a multiple of n_kvh
                 (q, K, V, T + 1, n_kvh, 0.1),  # rows != T * n_kvh
                 (q[:, :64], K, V, T, n_kvh, 0.1)):
        with pytest.raises(c.MxsError) as e:
            c.mxs_attn_decode(*args)
        assert e.value.status == 2
    assert c.mxs_launch_count() == n0
