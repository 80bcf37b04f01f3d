"""The rank-table comparison the GPU parity tests use (tests/gpu_util.compare_ranks).

Ranks must equal the fp64 oracle's.  The one accepted difference is an exchange of
retained directions between candidates whose energies tie at the selection boundary,
which the oracle breaks by its fixed order (lower module index, then lower j) and any
other correct implementation may break differently.  These cases plant wrong tables
(an off-by-one in a group without a tie, a slot moved to a module that holds no tied
candidate, a changed total) and check that each is rejected."""
import numpy as np

from oracle import allocate as OA
from tests import gpu_util as G


def fleet():
    # group 0: modules 0 and 1 have identical spectra (every candidate of one has a tied
    # twin in the other) and module 2 a clearly different one; group 1: modules 3 and 4
    # with distinct energies
    sig = np.array([
        [1.0, 0.5, 0.5, 0.1],
        [1.0, 0.5, 0.5, 0.1],
        [1.0, 0.05, 0.02, 0.01],
        [1.0, 0.9, 0.1, 0.05],
        [1.0, 0.3, 0.2, 0.1],
    ])
    r = np.array([4, 4, 4, 4, 4])
    group = np.array([0, 0, 0, 1, 1])
    return sig, r, group


def oracle(sig, r, group, num=1, den=2, floor=1):
    ranks, info = OA.spectral_ranks(sig, r, group, num, den, floor)
    return ranks, info


def test_equal_tables_pass():
    sig, r, group = fleet()
    ranks, info = oracle(sig, r, group)
    assert G.compare_ranks(ranks, ranks, info, sig, r, group, 1)


def test_tied_exchange_passes():
    sig, r, group = fleet()
    ranks, info = oracle(sig, r, group)
    assert info[0]["gap_rel"] == 0.0          # the budget of group 0 ends inside a tie
    # budget 6 = three floors + three of the four tied candidates (j = 1, 2 of modules
    # 0 and 1); the oracle's order takes module 0's two first
    assert ranks[:3].tolist() == [3, 2, 1]
    swapped = ranks.copy()
    swapped[0], swapped[1] = 2, 3              # one tied slot moved from module 0 to 1
    assert G.compare_ranks(swapped, ranks, info, sig, r, group, 1)


def test_off_by_one_in_group_without_tie_fails():
    sig, r, group = fleet()
    ranks, info = oracle(sig, r, group)
    assert info[1]["gap_rel"] > 1e-12
    bad = ranks.copy()
    bad[3] -= 1
    bad[4] += 1                                # same total, wrong module
    assert not G.compare_ranks(bad, ranks, info, sig, r, group, 1)


def test_slot_moved_to_untied_module_fails():
    sig, r, group = fleet()
    ranks, info = oracle(sig, r, group)
    bad = ranks.copy()
    bad[0] -= 1
    bad[2] += 1                                # module 2 holds no candidate at the boundary
    assert not G.compare_ranks(bad, ranks, info, sig, r, group, 1)


def test_changed_total_fails():
    sig, r, group = fleet()
    ranks, info = oracle(sig, r, group)
    bad = ranks.copy()
    bad[1] += 1                                # tied module, but one slot over budget
    assert not G.compare_ranks(bad, ranks, info, sig, r, group, 1)


def test_rank_below_floor_fails():
    sig, r, group = fleet()
    ranks, info = oracle(sig, r, group, floor=2)
    bad = ranks.copy()
    bad[0] -= 1
    bad[1] += 1
    if bad[0] >= 2:
        bad[0], bad[1] = 1, bad[1] + bad[0] - 1
    assert not G.compare_ranks(bad, ranks, info, sig, r, group, 2)
