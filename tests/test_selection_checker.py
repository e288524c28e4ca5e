"""The near-tie rule the GPU tests use to compare a device selection (top-C
of the token scores, a Deep Forcing region) with the fp64 selection.

Reading S1 (ii): against the fp64 top-C, a selection may swap only tokens
whose fp64 scores lie within the score tolerance of the C-th highest. These
checks plant the mistakes a selection kernel could make (a token far below
the cut kept, a clear winner dropped, a token kept twice, an index off by
one) and check each is caught, and that near-tie swaps pass.
"""
import numpy as np

from rcutil import SCORE_TOL, near_tie_violations


def _scores(n=400, seed=0):
    return np.random.default_rng(seed).random(n) * 5.0


def test_exact_selection_passes():
    s = _scores()
    C = 100
    want = np.sort(np.lexsort((np.arange(len(s)), -s))[:C])
    assert near_tie_violations(s, want, C) == []


def test_far_swap_is_caught():
    s = _scores()
    C = 100
    order = np.lexsort((np.arange(len(s)), -s))
    sel = list(order[:C])
    sel[0] = order[-1]                 # the best token replaced by the worst
    assert near_tie_violations(s, sel, C) != []


def test_second_of_the_cut_is_caught_unless_near_tie():
    s = _scores()
    C = 100
    order = np.lexsort((np.arange(len(s)), -s))
    sel = list(order[:C])
    sel[-1] = order[C]                 # the C-th swapped for the (C+1)-th
    gap = s[order[C - 1]] - s[order[C]]
    bad = near_tie_violations(s, sel, C)
    assert (bad == []) == (gap <= SCORE_TOL * max(1.0, s[order[C - 1]]))
    # make them a near-tie: now the swap is allowed
    s2 = s.copy()
    s2[order[C]] = s2[order[C - 1]] - 0.5 * SCORE_TOL
    assert near_tie_violations(s2, sel, C) == []


def test_duplicate_and_out_of_range_are_caught():
    s = _scores()
    C = 50
    order = np.lexsort((np.arange(len(s)), -s))
    dup = list(order[:C])
    dup[1] = dup[0]
    assert near_tie_violations(s, dup, C) != []
    off = list(order[:C])
    off[0] = len(s)                    # one past the last candidate
    assert near_tie_violations(s, off, C) != []


def test_exact_ties_allow_either_index():
    # exact ties at the cut: the fp64 rule keeps the lower index, a selection
    # keeping the higher one differs only by a tie and passes this check (the
    # exact tie order is checked bit for bit on the kernel's own scores)
    s = np.array([3.0, 2.0, 1.0, 1.0, 0.5])
    assert near_tie_violations(s, [0, 1, 2], 3) == []
    assert near_tie_violations(s, [0, 1, 3], 3) == []
    assert near_tie_violations(s, [0, 1, 4], 3) != []


def test_fewer_candidates_than_c():
    s = np.array([1.0, 2.0])
    assert near_tie_violations(s, [0, 1], 5) == []
    assert near_tie_violations(s, [0], 5) != []
