"""Pins for the oracle's bit allocation.

Closed forms from the budget arithmetic (including the pages' 4.03-bit
figure), an independent sort-based reformulation of the greedy, and
structural invariants of the permutation.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle


def _used_bits(K, N, counts):
    return sum(n * (4 * k + 4 * c[0] + 2 * c[1]) for k, n, c in zip(K, N, counts))


@pytest.mark.parametrize("K,N,budget,n6", [
    (4096, 4096, (129, 32), 0),       # 4.03125 bits: the fixed block only
    (4096, 4096, (9, 2), 960),
    (4096, 1024, (9, 2), 960),
    (14336, 4096, (9, 2), 3520),
    (8192, 8192, (17, 4), 960),
    (28672, 8192, (17, 4), 3520),
])
def test_single_layer_closed_form(K, N, budget, n6):
    s = np.random.default_rng(K).random(K)
    perms, counts = oracle.allocate([s], [N], mode="budget", budget=budget)
    assert tuple(counts[0]) == (32, n6, K - 32 - n6)
    # the budget is met with equality in these cases
    assert Fraction(_used_bits([K], [N], counts), N * K) == Fraction(*budget)


def test_pages_overhead_figure():
    # TS section 4: at ~4.03 bits about 1% of the work is at higher precision.
    # The fixed block alone costs 4 + 4*32/4096 = 4.03125 bits (printed as
    # 4.03), one 6-bit group adds 2*32/4096 = 0.015625: a 4.035 budget holds
    # the block and nothing more.
    s = np.random.default_rng(0).random(4096)
    with pytest.raises(ValueError):
        oracle.allocate([s], [4096], mode="budget", budget=(403, 100))
    _, counts = oracle.allocate([s], [4096], mode="budget", budget=(807, 200))
    n8, n6, n4 = counts[0]
    assert (n8, n6) == (32, 0)
    assert abs(n8 / 4096 - 0.01) < 0.003


def test_fractions_mode_counts():
    s = np.random.default_rng(0).random(256)
    _, counts = oracle.allocate([s], [256], mode="fractions", p8=(5, 100), p6=(15, 100))
    assert tuple(counts[0]) == (13, 38, 205)
    _, counts = oracle.allocate([np.ones(10)], [1], mode="fractions", p8=(1, 4), p6=(1, 4))
    assert tuple(counts[0]) == (3, 3, 4)        # 2.5 rounds half up to 3


def test_permutation_structure_and_ranking():
    rng = np.random.default_rng(5)
    K = 300
    s = rng.random(K)
    s[10] = s[20] = s[30] = 5.0                  # ties among the top
    perms, counts = oracle.allocate([s], [64], mode="budget", budget=(19, 4))
    perm = perms[0]
    n8, n6, n4 = counts[0]
    assert sorted(perm) == list(range(K))
    segs = [perm[:n8], perm[n8:n8 + n6], perm[n8 + n6:]]
    for seg in segs:
        assert np.all(np.diff(seg) > 0)
    order = sorted(range(K), key=lambda j: (-s[j], j))   # independent ranking
    assert set(segs[0]) == set(order[:n8])
    assert set(segs[1]) == set(order[n8:n8 + n6])
    assert n6 % 32 == 0


def test_ties_prefer_lower_index():
    perms, counts = oracle.allocate([np.zeros(1000)], [10], mode="budget", budget=(9, 2))
    n8, n6, _ = counts[0]
    assert (n8, n6) == (32, 160)
    assert list(perms[0][:n8]) == list(range(n8))
    assert list(perms[0][n8:n8 + n6]) == list(range(n8, n8 + n6))


def test_rank_order_matches_python_sort():
    s = np.random.default_rng(9).integers(0, 5, 200).astype(float)
    assert list(oracle.rank_order(s)) == sorted(range(200), key=lambda j: (-s[j], j))


def test_infeasible_budget():
    with pytest.raises(ValueError):
        oracle.allocate([np.ones(64)], [8], mode="budget", budget=(4, 1))


def _greedy_by_sorting(s_list, N, budget, w, fixed8=32):
    """Independent formulation: list every 32-column group of every layer,
    sort by gain/cost (exact rationals; ties: lower layer, then rank order),
    take the longest prefix whose cumulative cost fits."""
    num, den = budget
    cap = Fraction(num, den) * sum(n * len(s) for s, n in zip(s_list, N))
    used = Fraction(sum(n * (4 * len(s) + 4 * min(fixed8, len(s))) for s, n in zip(s_list, N)))
    groups = []
    for l, (s, n) in enumerate(zip(s_list, N)):
        order = sorted(range(len(s)), key=lambda j: (-s[j], j))
        n8 = min(fixed8, len(s))
        for gi, r0 in enumerate(range(n8, len(s), 32)):
            cols = order[r0:r0 + 32]
            gain = Fraction(w[l]) * sum(Fraction(float(s[j])) for j in cols)
            cost = 2 * n * len(cols)
            groups.append((-(gain / cost), l, gi, len(cols), cost))
    groups.sort()
    n6 = [0] * len(s_list)
    for _, l, _, cnt, cost in groups:
        if used + cost > cap:
            break
        used += cost
        n6[l] += cnt
    return n6


@pytest.mark.parametrize("seed", range(8))
def test_multi_layer_greedy_matches_sorted_prefix(seed):
    rng = np.random.default_rng(seed)
    L = int(rng.integers(2, 5))
    Ks = [int(rng.integers(200, 600)) for _ in range(L)]
    Ns = [int(rng.integers(1, 50)) for _ in range(L)]
    # integer-valued s keep the fp64 group sums exact, so the comparison with
    # exact rationals is a fair one
    s_list = [rng.integers(0, 1000, k).astype(float) * float(rng.integers(1, 9)) for k in Ks]
    w = [float(rng.integers(1, 4)) for _ in range(L)]
    budget = (int(rng.integers(19, 23)), 4)     # >= 4.75 bits: always feasible here
    perms, counts = oracle.allocate(s_list, Ns, mode="budget", budget=budget, layer_w=w)
    expect = _greedy_by_sorting(s_list, Ns, budget, w)
    assert list(counts[:, 1]) == expect
    assert Fraction(_used_bits(Ks, Ns, counts), sum(n * k for n, k in zip(Ns, Ks))) <= Fraction(*budget)


def test_layer_weight_steers_upgrades():
    # two layers of K=320, N=10: the fixed blocks cost 28160 bits, each 6-bit
    # group 640; a 4.65-bit budget (29760 bits) leaves room for two groups.
    s = [np.ones(320), np.ones(320)]
    _, c = oracle.allocate(s, [10, 10], mode="budget", budget=(93, 20), layer_w=[1.0, 3.0])
    assert list(c[:, 1]) == [0, 64]           # both go to the heavier layer
    _, c = oracle.allocate(s, [10, 10], mode="budget", budget=(93, 20), layer_w=[1.0, 1.0])
    assert list(c[:, 1]) == [64, 0]           # equal ratios: the lower layer wins each tie


# ------------------------------------------------ layer-score rule (mode 2)
def _r_rule_brute(K, N, scores, budget, fixed8=32):
    """The layer-score rule from its definition, with exact fractions: every
    R at which some layer's count changes (R = 32 k / w) is a candidate;
    n6_l(R) = min(K_l - n8_l, 32 floor(R w_l / 32)); the answer is the counts
    at the largest candidate R (or 0) whose counts meet the budget."""
    n8 = [min(fixed8, k) for k in K]
    cands = {Fraction(0)}
    for k, w, e in zip(K, scores, n8):
        if w > 0:
            for j in range(1, (k - e + 31) // 32 + 1):
                cands.add(Fraction(32 * j) / Fraction(w))
    best = None
    for R in sorted(cands):
        n6 = [min(k - e, 32 * int((R * Fraction(w)) // 32)) if w > 0 else 0 for k, w, e in zip(K, scores, n8)]
        used = sum(n * (4 * k + 4 * e + 2 * c) for k, n, e, c in zip(K, N, n8, n6))
        if Fraction(used, sum(n * k for k, n in zip(K, N))) <= Fraction(*budget):
            best = n6
        else:
            break
    return [(e, c, k - e - c) for k, e, c in zip(K, n8, best)]


def test_layer_rule_is_proportional_and_meets_the_budget():
    s = [np.random.default_rng(i).random(4096) for i in range(2)]
    _, counts = oracle.allocate(s, [4096, 4096], mode="layer", budget=(9, 2), layer_w=[2.0, 1.0])
    assert [tuple(c) for c in counts] == [(32, 1280, 2784), (32, 640, 3424)]
    assert Fraction(_used_bits([4096] * 2, [4096] * 2, counts), 2 * 4096 * 4096) == Fraction(9, 2)


@pytest.mark.parametrize("K,N,budget,n6", [
    (4096, 4096, (9, 2), 960), (14336, 4096, (9, 2), 3520), (8192, 8192, (17, 4), 960),
    (28672, 8192, (17, 4), 3520), (4096, 4096, (129, 32), 0)])
def test_layer_rule_single_layer_closed_form(K, N, budget, n6):
    # one layer: R only scales that layer, so the rule fills the budget
    s = np.random.default_rng(K).random(K)
    _, counts = oracle.allocate([s], [N], mode="layer", budget=budget, layer_w=[0.37])
    assert tuple(counts[0]) == (32, n6, K - 32 - n6)


def test_layer_rule_zero_score_and_ties():
    s = [np.random.default_rng(i).random(256) for i in range(3)]
    # a zero score gets no 6-bit columns; the others share the budget
    _, counts = oracle.allocate(s, [64, 64, 64], mode="layer", budget=(5, 1), layer_w=[1.0, 0.0, 1.0])
    assert counts[1][1] == 0 and counts[0][1] == counts[2][1] > 0
    # equal scores on equal layers step together: a budget with room for
    # three 32-column groups takes two (one each), never three
    K, N = [256, 256], [16, 16]
    used0 = sum(n * (4 * k + 4 * 32) for k, n in zip(K, N))
    room = used0 + 3 * 2 * 16 * 32
    _, counts = oracle.allocate([s[0], s[1]], N, mode="layer", budget=(room, sum(n * k for k, n in zip(K, N))),
                                layer_w=[0.5, 0.5])
    assert [c[1] for c in counts] == [32, 32]


@pytest.mark.parametrize("seed", range(6))
def test_layer_rule_matches_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    L = int(rng.integers(1, 5))
    K = [int(rng.choice([40, 64, 100, 130, 200])) for _ in range(L)]
    N = [int(rng.choice([8, 16, 24])) for _ in range(L)]
    scores = [float(rng.choice([0.0, rng.random(), rng.random() * 10, 1.0])) for _ in range(L)]
    budget = (int(rng.integers(41, 60)), 10)
    s = [rng.random(k) for k in K]
    try:
        _, counts = oracle.allocate(s, N, mode="layer", budget=budget, layer_w=scores)
    except ValueError:
        used = sum(n * (4 * k + 4 * min(32, k)) for k, n in zip(K, N))
        assert Fraction(used, sum(n * k for k, n in zip(K, N))) > Fraction(*budget)
        return
    assert [tuple(int(x) for x in c) for c in counts] == _r_rule_brute(K, N, scores, budget)
