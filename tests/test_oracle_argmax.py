"""Argmax rule of the oracle: ties to the lowest index, NaN never wins.

Greedy drafting and greedy verify take the argmax of a logit row (page
"FlashMap Drafts 16 Dependent Tokens at Once…", section "Why drafting still
costs time": the target's greedy choice decides).  Ties go to the lowest
index; a NaN entry ranks below every number, -inf included; a row of NaN
gives index 0.  The CUDA kernels follow the same rule.
"""
import numpy as np

from oracle import flashmap as fm


def test_ties_go_to_the_lowest_index():
    assert fm.argmax_lowest(np.array([1.0, 3.0, 3.0, 2.0])) == 1
    assert fm.argmax_lowest(np.zeros(7)) == 0
    assert fm.argmax_lowest(np.full(5, -np.inf)) == 0


def test_nan_never_wins():
    nan, inf = np.nan, np.inf
    assert fm.argmax_lowest(np.array([nan, 1.0, 2.0])) == 2
    assert fm.argmax_lowest(np.array([1.0, nan, 1.0])) == 0
    assert fm.argmax_lowest(np.array([nan, -inf, -inf])) == 1   # below -inf too
    assert fm.argmax_lowest(np.array([nan, nan])) == 0


def test_greedy_verify_skips_nan():
    K, V = 2, 4
    t = np.zeros((1, K + 1, V))
    t[0, 0] = [np.nan, 5.0, 1.0, 5.0]          # argmax 1 (NaN skipped, tie -> lowest)
    t[0, 1] = [np.nan, np.nan, np.nan, np.nan]  # all NaN -> 0
    t[0, 2] = [0.0, np.nan, 9.0, 1.0]
    n, b, out = fm.verify_greedy(t, [[1, 0]])
    assert (n, b, out) == (2, 0, [1, 0, 2])
