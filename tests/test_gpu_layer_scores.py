"""GPU parity: mxs_layer_scores against the oracle's fp64 decoder-stack
forward, and the layer-score allocation on the Llama-3-8B 224-matrix stack.

Scores are compared per layer with relative tolerance SCORE_RTOL.  The GPU
runs the unquantised stack in fp32 against the oracle's fp64, so its outputs
differ by about 1e-6 relative; a score is the norm of the difference between
two outputs, 1-10% of their size here, so the fp32 noise moves it by about
1e-4 relative.  A code of the quantised layer's input or a bf16 rounding of
its output can also land on the other side of a tie between the two
computations; each such flip moves one element by one step, well under the
budget at these sizes.  The allocation built on the scores is integer work:
given the same scores, GPU and oracle counts and permutations must be equal.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import stack
from mx_microscaling_mixed_b200 import inputs
from tests import parity

pytestmark = pytest.mark.gpu

SCORE_RTOL = 1e-3


@pytest.fixture(scope="module")
def c():
    parity.need_gpu()
    return parity.capi()


def _shapes(hidden, H, G, mlp):
    d = hidden // H
    return [(H * d, hidden), (G * d, hidden), (G * d, hidden), (hidden, H * d), (mlp, hidden), (mlp, hidden),
            (hidden, mlp)]


def _stack(seed, n_blocks, hidden, H, G, mlp):
    # the workload's weight recipe: N(0, 0.02^2) with 3% Student-t(3) columns, bf16
    return [tuple(inputs.attn_weight("cuda", seed + 16 * b + j, n, k) for j, (n, k) in
                  enumerate(_shapes(hidden, H, G, mlp))) for b in range(n_blocks)]


def _oracle_scores(x, blocks, hidden, H, G, mlp, theta, layers=None):
    cfg = stack.StackConfig(hidden=hidden, n_heads=H, n_kv_heads=G, mlp=mlp, rope_theta=theta)
    hb = [tuple(parity.host64(w) for w in Ws) for Ws in blocks]
    return stack.layer_scores(parity.host64(x), hb, cfg, layers)


@pytest.mark.parametrize("T,n_blocks,hidden,H,G,mlp", [
    (24, 2, 256, 4, 2, 512),       # ragged token tile, grouped heads
    (80, 2, 256, 8, 8, 384),       # two token tiles, one query head per kv head
    (8, 3, 128, 2, 1, 256),        # few tokens: the quantised product takes the decode kernels
])
def test_scores_match_oracle(c, T, n_blocks, hidden, H, G, mlp):
    theta = 10000.0
    blocks = _stack(500 + T, n_blocks, hidden, H, G, mlp)
    x = inputs.gaussian_acts("cuda", 900 + T, T, hidden).float()
    got = c.mxs_layer_scores(x, blocks, n_heads=H, n_kv_heads=G, rope_theta=theta)
    want = _oracle_scores(x, blocks, hidden, H, G, mlp, theta)
    rel = np.abs(got - want) / want
    print(f"T={T} blocks={n_blocks} hidden={hidden}: max rel err {rel.max():.2e}, scores {want.min():.3g}..{want.max():.3g}")
    assert np.all(want > 0) and rel.max() <= SCORE_RTOL


def test_llama3_dims_sampled_layers(c):
    """Llama-3-8B block dimensions (hidden 4096, 32/8 heads, MLP 14336), two
    blocks, 16 tokens: three layers checked against the oracle."""
    T, hidden, H, G, mlp = 16, 4096, 32, 8, 14336
    blocks = _stack(700, 2, hidden, H, G, mlp)
    x = inputs.gaussian_acts("cuda", 701, T, hidden).float()
    got = c.mxs_layer_scores(x, blocks, n_heads=H, n_kv_heads=G)
    layers = [0, 3, 13]
    want = _oracle_scores(x, blocks, hidden, H, G, mlp, 500000.0, layers)
    rel = np.abs(got[layers] - want) / want
    print(f"llama3 dims: rel err {rel}")
    assert rel.max() <= SCORE_RTOL


def test_stack_224_layer_allocation(c):
    """The whole random-init Llama-3-8B stack (32 blocks, 224 matrices): GPU
    layer scores feed MXS_ALLOC_LAYER under a 4.5-bit budget; counts and
    permutations equal the oracle's rule on the same scores, and the budget
    holds across the stack."""
    T, hidden, H, G, mlp = 8, 4096, 32, 8, 14336
    blocks = _stack(1000, 32, hidden, H, G, mlp)
    x = inputs.gaussian_acts("cuda", 1001, T, hidden).float()
    scores = c.mxs_layer_scores(x, blocks, n_heads=H, n_kv_heads=G)
    assert scores.shape == (224,) and np.all(np.isfinite(scores)) and np.all(scores > 0)
    shapes = _shapes(hidden, H, G, mlp) * 32
    Ns = [n for n, _ in shapes]
    rng = np.random.default_rng(9)
    s_np = [rng.standard_t(3, k) ** 2 for _, k in shapes]
    s_dev = [torch.from_numpy(v).cuda() for v in s_np]
    gp, gc = c.mxs_allocate(s_dev, Ns, mode="layer", budget=(9, 2), layer_w=list(scores))
    op, oc = oracle.allocate(s_np, Ns, mode="layer", budget=(9, 2), layer_w=scores)
    for l in range(224):
        assert tuple(gc[l]) == tuple(int(v) for v in oc[l]), l
        assert np.array_equal(gp[l].cpu().numpy(), op[l]), l
    bits = sum(n * (8 * a + 6 * b + 4 * d) for n, (a, b, d) in zip(Ns, gc))
    assert bits <= 4.5 * sum(n * k for n, k in shapes)
    # more sensitive layers get at least as many 6-bit columns, per column
    # of room (n6 / w is the same R for every layer not at its cap)
    frac = [gc[l][1] / scores[l] for l in range(224) if 0 < gc[l][1] < shapes[l][1] - 32]
    assert max(frac) - min(frac) <= 32 / min(scores) + 1e-9
