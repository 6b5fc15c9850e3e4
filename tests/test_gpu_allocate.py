"""GPU parity: mxs_allocate (ranking, counts, permutation) against the
oracle, exactly; the sensitivity feeding it is the GPU's own on one side and
the oracle's on the other (they are bit-identical)."""
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


def _cmp(gp, gc, op, oc):
    for l in range(len(op)):
        assert tuple(gc[l]) == tuple(int(x) for x in oc[l]), l
        assert np.array_equal(gp[l].cpu().numpy(), op[l]), l


def test_parity_layer_fractions(c):
    d = inputs.parity_layer("cuda", seed=0)
    _, _, s = c.mxs_sensitivity(d["X"], d["W"])
    gp, gc = c.mxs_allocate([s], [256], mode="fractions", p8=(5, 100), p6=(15, 100))
    _, _, so = oracle.sensitivity(parity.host64(d["X"]), parity.host64(d["W"]))
    op, oc = oracle.allocate([so], [256], mode="fractions", p8=(5, 100), p6=(15, 100))
    assert tuple(gc[0]) == (13, 38, 205)
    _cmp(gp, gc, op, oc)


def test_attention_layer_budget(c):
    X = inputs.gaussian_acts("cuda", seed=2001, rows=512, K=4096)
    W = inputs.attn_weight("cuda", seed=2000, N=1024)
    _, _, s = c.mxs_sensitivity(X, W)
    gp, gc = c.mxs_allocate([s], [1024], mode="budget", budget=(9, 2))
    _, _, so = oracle.sensitivity(parity.host64(X), parity.host64(W))
    op, oc = oracle.allocate([so], [1024], mode="budget", budget=(9, 2))
    assert tuple(gc[0]) == (32, 960, 3104)
    _cmp(gp, gc, op, oc)


@pytest.mark.parametrize("seed", range(4))
def test_multi_layer_budget(c, seed):
    rng = np.random.default_rng(seed)
    L = 5
    Ks = [int(k) for k in rng.integers(300, 3000, L)]
    Ns = [int(n) for n in rng.integers(16, 512, L)]
    # integer-valued sensitivities make ties across and within layers common
    s_np = [rng.integers(0, 50, k).astype(np.float64) * 0.5 for k in Ks]
    w = [float(x) for x in rng.integers(1, 4, L)]
    s_dev = [torch.from_numpy(x).cuda() for x in s_np]
    gp, gc = c.mxs_allocate(s_dev, Ns, mode="budget", budget=(19, 4), layer_w=w)
    op, oc = oracle.allocate(s_np, Ns, mode="budget", budget=(19, 4), layer_w=w)
    _cmp(gp, gc, op, oc)


def test_all_ties(c):
    s = torch.zeros(1000, dtype=torch.float64, device="cuda")
    gp, gc = c.mxs_allocate([s], [10], mode="budget", budget=(9, 2))
    op, oc = oracle.allocate([np.zeros(1000)], [10], mode="budget", budget=(9, 2))
    _cmp(gp, gc, op, oc)


def test_large_k(c):
    s_np = np.random.default_rng(3).random(28672)
    s = torch.from_numpy(s_np).cuda()
    gp, gc = c.mxs_allocate([s], [8192], mode="budget", budget=(17, 4))
    op, oc = oracle.allocate([s_np], [8192], mode="budget", budget=(17, 4))
    assert tuple(gc[0]) == (32, 3520, 28672 - 3552)
    _cmp(gp, gc, op, oc)


def test_large_k_ties(c):
    """Long rows with heavy ties: four distinct values, -0.0 among the zeros
    (equal to +0.0, so the two must tie and fall back to the column index),
    the 8/6/4 boundaries inside tie groups; one layer in fractions mode and two
    in the multi-layer budget greedy (whose group gains follow the rank
    order)."""
    rng = np.random.default_rng(21)
    s_np = rng.integers(0, 4, 16384).astype(np.float64)
    s_np[rng.random(16384) < 0.1] = -0.0
    s_np[s_np == 0] = np.where(rng.random(int((s_np == 0).sum())) < 0.5, 0.0, -0.0)
    s = torch.from_numpy(s_np).cuda()
    gp, gc = c.mxs_allocate([s], [100], mode="fractions", p8=(7, 100), p6=(31, 100))
    op, oc = oracle.allocate([s_np], [100], mode="fractions", p8=(7, 100), p6=(31, 100))
    _cmp(gp, gc, op, oc)
    t_np = np.round(rng.random(9000) * 50) / 8                       # 401 distinct values
    s2 = [s, torch.from_numpy(t_np).cuda()]
    gp, gc = c.mxs_allocate(s2, [300, 500], mode="budget", budget=(19, 4))
    op, oc = oracle.allocate([s_np, t_np], [300, 500], mode="budget", budget=(19, 4))
    _cmp(gp, gc, op, oc)


def test_infeasible_budget(c):
    s = torch.ones(64, dtype=torch.float64, device="cuda")
    with pytest.raises(c.MxsError) as e:
        c.mxs_allocate([s], [8], mode="budget", budget=(4, 1))
    assert e.value.status == 5


def test_llama3_8b_stack_global_budget(c):
    """The whole Llama-3-8B linear stack under one 4.5-bit budget: 32 layers x
    (q, k, v, o 4096-wide inputs; gate, up 4096; down 14336), layer weights the
    output widths' shares, one greedy across all 224 layers."""
    rng = np.random.default_rng(8)
    shapes = [(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096), (14336, 4096), (14336, 4096),
              (4096, 14336)] * 32                      # (N, K) per layer
    Ns = [n for n, _ in shapes]
    # heavy-tailed sensitivities with per-layer scale, as outlier columns give
    s_np = [rng.standard_t(3, k) ** 2 * float(rng.uniform(0.5, 2.0)) for _, k in shapes]
    s_dev = [torch.from_numpy(x).cuda() for x in s_np]
    gp, gc = c.mxs_allocate(s_dev, Ns, mode="budget", budget=(9, 2))
    op, oc = oracle.allocate(s_np, Ns, mode="budget", budget=(9, 2))
    _cmp(gp, gc, op, oc)
    bits = sum(n * (8 * a + 6 * b + 4 * d) for n, (a, b, d) in zip(Ns, gc))
    elems = sum(n * k for n, k in shapes)
    assert bits <= 4.5 * elems                          # the budget holds across the stack


@pytest.mark.parametrize("seed", range(3))
def test_layer_score_rule(c, seed):
    """MXS_ALLOC_LAYER: 6-bit counts proportional to the layer scores under one
    global R; counts and permutations exact against the oracle, including
    zero scores and repeated scores (steps taken together)."""
    rng = np.random.default_rng(40 + seed)
    L = 6
    Ks = [int(k) for k in rng.integers(100, 5000, L)]
    Ns = [int(n) for n in rng.integers(16, 1024, L)]
    s_np = [rng.integers(0, 50, k).astype(np.float64) * 0.25 for k in Ks]
    w = [float(x) for x in rng.choice([0.0, 0.5, 1.0, 1.0, 2.75, float(rng.random())], L)]
    s_dev = [torch.from_numpy(x).cuda() for x in s_np]
    n0 = c.mxs_launch_count()
    gp, gc = c.mxs_allocate(s_dev, Ns, mode="layer", budget=(9, 2), layer_w=w)
    op, oc = oracle.allocate(s_np, Ns, mode="layer", budget=(9, 2), layer_w=w)
    _cmp(gp, gc, op, oc)
    assert c.mxs_launch_count() - n0 == 2 * L             # rank + placement per layer, no gains pass
    with pytest.raises(c.MxsError) as e:
        c.mxs_allocate(s_dev, Ns, mode="layer", budget=(9, 2), layer_w=None)
    assert e.value.status == 1
