"""Pins for oracle.allocate: hand-worked fixtures, brute force, invariants."""
import json
import math
import os

import numpy as np
import pytest

from oracle import allocate as AL
from tests.conftest import GOLDEN

GOLD = json.load(open(os.path.join(GOLDEN, "allocation_cases.json")))


@pytest.mark.parametrize("case", GOLD["uniform"])
def test_uniform_closed_form(case):
    assert AL.uniform_rank(case["r"], case["num"], case["den"], case["floor"]) == case["k"]


@pytest.mark.parametrize("case", GOLD["spectral"], ids=[c["name"] for c in GOLD["spectral"]])
def test_spectral_hand_cases(case):
    ranks, info = AL.spectral_ranks(np.array(case["sigma"], dtype=float), case["r"], case["group"],
                                    case["num"], case["den"], case["floor"])
    assert ranks.tolist() == case["ranks"]


def test_below_floor_flagged():
    case = [c for c in GOLD["spectral"] if c["name"] == "below-floor-budget"][0]
    _, info = AL.spectral_ranks(np.array(case["sigma"], float), case["r"], case["group"],
                                case["num"], case["den"], case["floor"])
    assert info[0]["over_budget"]


def random_sigma(g, n, r):
    s = np.sort(np.abs(g.standard_normal((n, r))) * g.uniform(0.1, 3, size=(n, 1)), axis=1)[:, ::-1]
    return s


@pytest.mark.parametrize("seed", range(12))
def test_greedy_equals_brute_force(seed):
    g = np.random.default_rng(100 + seed)
    n, r = int(g.integers(2, 5)), 4
    sig = random_sigma(g, n, r)
    num, den = int(g.integers(1, 4)), 4
    floor = int(g.integers(1, 3))
    ranks, _ = AL.spectral_ranks(sig, [r] * n, [0] * n, num, den, floor)
    best, opts = AL.brute_force_ranks(sig, [r] * n, num, den, floor)
    E = [AL.energies(sig[i], r) for i in range(n)]
    val = sum(E[i][:ranks[i]].sum() for i in range(n))
    assert val == pytest.approx(best, abs=1e-12)
    assert tuple(int(k) for k in ranks) in opts


@pytest.mark.parametrize("seed", range(6))
def test_invariants_and_monotone(seed):
    g = np.random.default_rng(200 + seed)
    n, r = 30, 16
    sig = random_sigma(g, n, r)
    grp = np.repeat([0, 1, 2], 10)
    prev = None
    for num in range(1, 13):
        ranks, info = AL.spectral_ranks(sig, [r] * n, grp, num, 12, 1)
        assert np.all(ranks >= 1) and np.all(ranks <= r)
        for gi in range(3):
            K = (num * r * 10) // 12
            assert ranks[grp == gi].sum() <= max(K, 10)
        if prev is not None:
            assert np.all(ranks >= prev)  # more budget never lowers a rank
        prev = ranks


def test_prefix_closed_with_ties():
    # equal energies inside one module are taken in j order
    sig = np.array([[2.0, 1.0, 1.0, 1.0, 1.0]])
    for num in range(1, 6):
        ranks, _ = AL.spectral_ranks(sig, [5], [0], num, 5, 1)
        assert ranks[0] == max(1, num)


def test_rejects_unsorted_sigma():
    with pytest.raises(ValueError):
        AL.spectral_ranks(np.array([[1.0, 2.0, 0.5]]), [3], [0], 1, 2, 1)


def test_absolute_energy_variant_hand_case():
    # module 0: sigma (10, 1), module 1: sigma (1, 0.9); K = floor(3 * 4 / 4) = 3,
    # floor 1 -> one extra slot.  Normalised energies of the second directions:
    # 1/101 = 0.0099 vs 0.81/1.81 = 0.4475 -> module 1 gets it.  Absolute energies:
    # 1.0 vs 0.81 -> module 0 gets it.
    sig = np.array([[10.0, 1.0], [1.0, 0.9]])
    rk_norm, _ = AL.spectral_ranks(sig, [2, 2], [0, 0], 3, 4, 1)
    rk_abs, _ = AL.spectral_ranks(sig, [2, 2], [0, 0], 3, 4, 1, absolute=True)
    assert rk_norm.tolist() == [1, 2]
    assert rk_abs.tolist() == [2, 1]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_absolute_energy_variant_minimises_dense_truncation_error(seed):
    # the definition: among all rank vectors within the budget, the variant's ranks
    # minimise sum_i ||dW_i - best rank-k_i approximation||_F^2, evaluated here from
    # dense SVDs of dW_i = B_i A_i (no energies involved)
    g = np.random.default_rng(seed)
    mods = []
    for _ in range(3):
        B = g.standard_normal((9, 4)) * np.exp(g.standard_normal(4))
        A = g.standard_normal((4, 7))
        mods.append(B @ A)
    sig = np.stack([np.linalg.svd(W, compute_uv=False)[:4] for W in mods])
    rk, _ = AL.spectral_ranks(sig, [4] * 3, [0] * 3, 1, 2, 1, absolute=True)

    def err(ks):
        tot = 0.0
        for W, k in zip(mods, ks):
            U, s, Vt = np.linalg.svd(W, full_matrices=False)
            tot += np.linalg.norm(W - (U[:, :k] * s[:k]) @ Vt[:k]) ** 2
        return tot
    import itertools
    K = (1 * 12) // 2
    best = min(err(ks) for ks in itertools.product(range(1, 5), repeat=3) if sum(ks) <= K)
    assert err(rk) <= best * (1 + 1e-12) + 1e-12
    assert int(rk.sum()) <= K


def test_absolute_energy_brute_force_agrees():
    g = np.random.default_rng(7)
    sig = np.sort(np.exp(g.standard_normal((4, 4))), axis=1)[:, ::-1]
    rk, _ = AL.spectral_ranks(sig, [4] * 4, [0] * 4, 1, 2, 1, absolute=True)
    best, args = AL.brute_force_ranks(sig, [4] * 4, 1, 2, 1, absolute=True)
    assert tuple(rk.tolist()) in [tuple(a) for a in args]


# ---- energy fraction (LoRASpace's minimal subspace keeping a fraction of the energy) ----

def test_energy_fraction_hand_case():
    # sigma = 3, 2, 1: energies 9, 4, 1 of 14
    s = [3.0, 2.0, 1.0]
    assert AL.energy_fraction_rank(s, 3, 1, 2, 1)[0] == 1        # 9 >= 7
    assert AL.energy_fraction_rank(s, 3, 9, 10, 1)[0] == 2       # 13 >= 12.6 > 9
    assert AL.energy_fraction_rank(s, 3, 19, 20, 1)[0] == 3      # 13 < 13.3
    assert AL.energy_fraction_rank(s, 3, 13, 14, 1)[0] == 2      # exactly 13/14: the tie keeps k = 2
    assert AL.energy_fraction_rank(s, 3, 1, 100, 2)[0] == 2      # the floor
    assert AL.energy_fraction_rank([2.0, 1.0, 0.0, 0.0], 4, 1, 1, 1)[0] == 2   # all of it: last nonzero
    assert AL.energy_fraction_rank([0.0, 0.0], 2, 99, 100, 1)[0] == 1          # zero module: floor


def test_energy_fraction_geometric_closed_form():
    # sigma_j^2 = q^j (j = 0..r-1): the leading-k fraction is (1 - q^k) / (1 - q^r), so the
    # smallest k reaching rho is ceil(log(1 - rho (1 - q^r)) / log q)
    for q, r, num, den in [(0.5, 20, 99, 100), (0.8, 32, 9, 10), (0.9, 64, 99, 100), (0.7, 16, 1, 3)]:
        s = np.sqrt(q ** np.arange(r))
        rho = num / den
        want = math.ceil(math.log(1 - rho * (1 - q ** r)) / math.log(q) - 1e-12)
        assert AL.energy_fraction_rank(s, r, num, den, 1)[0] == max(1, want), (q, r, num, den)


def test_energy_fraction_is_monotone_and_keeps_the_fraction():
    g = np.random.default_rng(21)
    for _ in range(50):
        r = int(g.integers(1, 40))
        s = np.sort(np.abs(g.standard_normal(r)) * np.exp(g.standard_normal(r)))[::-1]
        fl = int(g.integers(1, r + 1))
        prev = 0
        for num in range(0, 101, 5):
            k, _ = AL.energy_fraction_rank(s, r, num, 100, fl)
            assert fl <= k <= r and k >= prev
            prev = k
            e = s * s
            kept = e[:k].sum() / e.sum()
            assert kept >= num / 100 - 1e-12
            if k > fl:   # one direction fewer would not reach the fraction
                assert e[:k - 1].sum() / e.sum() < num / 100 + 1e-12
