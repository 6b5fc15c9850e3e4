"""GPU parity: mxs_quantize_weight / mxs_quantize_act / mxs_dequantize against
the oracle, byte for byte (codes and E8M0 scales)."""
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


def _random_layout(c, K, seed, counts=None):
    rng = np.random.default_rng(seed)
    if counts is None:
        n8 = int(rng.integers(0, K // 3 + 1))
        n6 = int(rng.integers(0, (K - n8) // 2 + 1))
        counts = (n8, n6, K - n8 - n6)
    perm = rng.permutation(K).astype(np.int32)
    lay = c.mxs_layout_make(K, counts, torch.from_numpy(perm).cuda())
    return lay, perm, counts


def _edge_matrix(rows, K, dtype, seed):
    """Row r takes pattern r % 8: zeros, fp32 subnormals, exact powers of two,
    half-step ties, huge magnitudes, negative block maxima, blocks just above
    the smallest normal scale with subnormal neighbours (where the scaled
    subnormals decide codes), and a different random scale per block."""
    g = torch.Generator().manual_seed(seed)
    X = torch.randn(rows, K, generator=g)
    nbk = (K + 31) // 32
    for r in range(rows):
        kind = r % 8
        if kind == 0:
            X[r] = 0.0
        elif kind == 1:
            X[r] = torch.randn(K, generator=g) * 1e-40          # subnormal (bf16 shares fp32's exponent range)
        elif kind == 2:
            X[r] = 2.0 ** torch.randint(-20, 20, (K,), generator=g).float()
        elif kind == 3:
            X[r] = (torch.randint(-60, 60, (K,), generator=g).float() + 0.5) * 2.0 ** -6
        elif kind == 4:
            X[r] = torch.randn(K, generator=g) * 1e37
        elif kind == 5:
            X[r] = -torch.rand(K, generator=g) - 1.0
        elif kind == 6:
            e = torch.randint(-127, -119, (nbk,), generator=g).float().repeat_interleave(32)[:K]
            x = torch.randn(K, generator=g) * 2.0 ** e
            sub = torch.rand(K, generator=g) < 0.5
            x[sub] = torch.randint(-127, 128, (int(sub.sum()),), generator=g).float() * 2.0 ** -133
            X[r] = x
        else:
            e = torch.randint(-130, 120, (nbk,), generator=g).float().repeat_interleave(32)[:K]
            X[r] = torch.randn(K, generator=g) * 2.0 ** e
    return X.to(dtype)


CASES = [
    # rows, K, dtype, counts (None = random), kind
    (256, 256, torch.float32, (13, 38, 205), "parity"),
    (37, 70, torch.float32, None, "random"),
    (37, 70, torch.bfloat16, None, "random"),
    (9, 1000, torch.bfloat16, None, "edge"),
    (9, 1000, torch.float32, None, "edge"),
    (8, 14336, torch.bfloat16, (32, 3520, 10784), "random"),
    (3, 30000, torch.float32, (32, 960, 29008), "random"),   # too large to stage: direct path
    (5, 33, torch.bfloat16, (1, 0, 32), "random"),
    (64, 4096, torch.bfloat16, (32, 960, 3104), "random"),
    (320, 1024, torch.bfloat16, None, "edge"),               # staged path (more than 8192 blocks)
    (320, 1024, torch.float32, None, "edge"),
    (333, 1000, torch.bfloat16, None, "random"),             # ragged last batch and last piece
    (1001, 520, torch.bfloat16, None, "edge"),               # odd rows: a lone row in the last pair
    (2048, 4096, torch.bfloat16, (32, 960, 3104), "random"),  # the attention projection's activations
]


@pytest.mark.parametrize("rows,K,dtype,counts,kind", CASES)
def test_quantize_matches_oracle(c, rows, K, dtype, counts, kind):
    if kind == "parity":
        src = inputs.parity_layer("cuda", seed=0)["W"]
    elif kind == "edge":
        src = _edge_matrix(rows, K, dtype, seed=K).cuda()
    else:
        src = inputs.random_matrix(rows, K, device="cuda", seed=rows * 7 + K, dtype=dtype)
    lay, perm, counts = _random_layout(c, K, seed=K + rows, counts=counts)
    for weight in (True, False):
        t, oc, os_ = parity.quantize_both(c, src, lay, perm, counts, weight)
        torch.cuda.synchronize()
        parity.assert_codes_equal(t, oc, os_, what=f"{kind} weight={weight}")


def test_strided_rows_staged(c):
    wide = inputs.random_matrix(400, 1024, device="cuda", seed=5, dtype=torch.bfloat16)
    src = wide[:, :1000]                     # pitch 1024 elements, K = 1000, staged path
    lay, perm, counts = _random_layout(c, 1000, seed=6)
    t, oc, os_ = parity.quantize_both(c, src, lay, perm, counts, weight=True)
    parity.assert_codes_equal(t, oc, os_, "strided staged")


@pytest.mark.parametrize("rows,K,counts,weight", [
    (300, 24008, (32, 5000, 18976), True),      # bf16 rows too wide for the gather table: offsets from the permutation
    (37, 28672, (32, 3520, 25120), False),      # the 70B down-projection width, a ragged row count
    (64, 24008, (7, 1001, 23000), True),        # segment starts off the 16-byte grid: single-entry loads
])
def test_wide_rows_table_free(c, rows, K, counts, weight):
    src = inputs.random_matrix(rows, K, device="cuda", seed=K + rows, dtype=torch.bfloat16)
    lay, perm, counts = _random_layout(c, K, seed=rows, counts=counts)
    t, oc, os_ = parity.quantize_both(c, src, lay, perm, counts, weight=weight)
    parity.assert_codes_equal(t, oc, os_, f"{rows} x {K} bf16")


def test_strided_rows(c):
    wide = inputs.random_matrix(20, 300, device="cuda", seed=3, dtype=torch.bfloat16)
    src = wide[:, :257]                      # pitch 300 elements, K = 257
    lay, perm, counts = _random_layout(c, 257, seed=4)
    t, oc, os_ = parity.quantize_both(c, src, lay, perm, counts, weight=False)
    parity.assert_codes_equal(t, oc, os_, "strided")


@pytest.mark.parametrize("rows,K", [(65536, 128), (1000, 96), (7, 33)])
def test_kv_identity_layout(c, rows, K):
    src = inputs.random_matrix(rows, K, device="cuda", seed=rows, dtype=torch.bfloat16, outlier_frac=0.0)
    lay = c.mxs_layout_make(K, (0, 0, K))
    t = c.mxtensor_empty(rows, lay)
    c.mxs_quantize_act(src, t)
    oc, os_ = oracle.quantize_rows(parity.host64(src), None, (0, 0, K))
    parity.assert_codes_equal(t, oc, os_, "kv")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_identity_layout_edge(c, dtype):
    """Unpermuted mixed layout on the direct path, edge values in every width."""
    rows, K, counts = 320, 1024, (96, 200, 728)
    src = _edge_matrix(rows, K, dtype, seed=5).cuda()
    lay = c.mxs_layout_make(K, counts)
    t = c.mxtensor_empty(rows, lay)
    c.mxs_quantize_act(src, t)
    oc, os_ = oracle.quantize_rows(parity.host64(src), None, counts)
    parity.assert_codes_equal(t, oc, os_, "identity edge")


def test_kv_cache_shape(c):
    kv = inputs.kv_cache("cuda", tokens=1024)             # tokens x heads x head_dim
    flat = kv.reshape(-1, kv.shape[-1])
    lay = c.mxs_layout_make(128, (0, 0, 128))
    t = c.mxtensor_empty(flat.shape[0], lay)
    c.mxs_quantize_act(flat, t)
    oc, os_ = oracle.quantize_rows(parity.host64(flat), None, (0, 0, 128))
    parity.assert_codes_equal(t, oc, os_, "kv cache")


def test_dequantize_matches_oracle(c):
    src = inputs.random_matrix(50, 200, device="cuda", seed=11, dtype=torch.float32)
    lay, perm, counts = _random_layout(c, 200, seed=12)
    t, oc, os_ = parity.quantize_both(c, src, lay, perm, counts, weight=True)
    deq = c.mxs_dequantize(t).cpu().numpy().astype(np.float64)
    assert np.array_equal(deq, oracle.dequantize_rows(oc, os_, counts))


def test_full_attention_weight(c):
    W = inputs.attn_weight("cuda", seed=2000)
    lay, perm, counts = _random_layout(c, 4096, seed=5, counts=(32, 960, 3104))
    t, oc, os_ = parity.quantize_both(c, W, lay, perm, counts, weight=True)
    parity.assert_codes_equal(t, oc, os_, "attn W 4096x4096")


def test_empty_rows(c):
    lay = c.mxs_layout_make(64, (0, 0, 64))
    t = c.mxtensor_empty(0, lay)
    c.mxs_quantize_act(torch.empty(0, 64, dtype=torch.bfloat16, device="cuda"), t)
    c.mxs_sync()
