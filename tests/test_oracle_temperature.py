"""Temperature scaling of the oracle's sampling and verify, pinned to closed forms.

Sampling at temperature T draws from softmax(logits / T) (page
"FlashMap并行草拟加速大模型解码", section "能拿来做什么": probabilistic draft
sampling for T > 0).  With two tokens the inverse CDF picks token 0 exactly
when u < sigmoid((z0 - z1) / T); with a point-mass draft, stochastic verify
accepts exactly when u < softmax(target / T)(y).  At T = 1 dividing and
multiplying by T agree, so every case here uses T != 1.
"""
import math

import numpy as np
import pytest

from oracle import flashmap as fm


@pytest.mark.parametrize("T", [0.25, 0.7, 2.0, 5.0])
@pytest.mark.parametrize("dz", [0.3, -1.1, 2.0])
def test_two_token_sampling_threshold(T, dz):
    z = np.array([1.5 + dz, 1.5])
    p0 = 1.0 / (1.0 + math.exp(-dz / T))          # sigmoid((z0 - z1) / T)
    assert fm.sample_row(z, T, p0 * (1 - 1e-9)) == 0
    assert fm.sample_row(z, T, p0 + 1e-9 * (1 - p0)) == 1


@pytest.mark.parametrize("T", [0.5, 3.0])
def test_three_token_sampling_cells(T):
    z = [0.4, -1.3, 1.1]
    e = [math.exp(a / T) for a in z]
    tot = sum(e)
    c0, c1 = e[0] / tot, (e[0] + e[1]) / tot
    for u, want in ((0.5 * c0, 0), (0.5 * (c0 + c1), 1), (0.5 * (c1 + 1.0), 2)):
        assert fm.sample_row(np.array(z), T, u) == want


@pytest.mark.parametrize("T", [0.6, 2.5])
def test_point_mass_draft_accepts_below_tempered_probability(T):
    V, K = 4, 2
    tgt = np.array([[0.2, 1.0, -0.5, 0.3], [0.0, 0.0, 0.0, 0.0], [1.0, 2.0, 3.0, 4.0]])
    e = [math.exp(a / T) for a in tgt[0]]
    p_y = e[1] / sum(e)                            # softmax(target / T) at y = 1
    for u, acc in ((p_y * 0.999, True), (p_y * 1.001, False)):
        ua = np.array([[u, 0.999999]])
        n, _, toks = fm.verify_sample(tgt[None], None, [[1, 2]], T, ua, 0.5)
        assert (n >= 1) == acc
        if not acc:
            assert toks[0] != 1


@pytest.mark.parametrize("T", [0.6, 2.5])
def test_draft_distribution_accept_ratio(T):
    # with a full draft distribution q, position 1 is accepted iff u q(y) < p(y)
    tgt = np.array([[0.2, 1.0, -0.5], [0.0, 0.0, 0.0], [0.0, 0.0, 0.0]])
    dl = np.array([[1.5, 0.1, 0.3], [0.0, 0.0, 0.0]])
    p = np.exp(tgt[0] / T) / np.exp(tgt[0] / T).sum()
    q = np.exp(dl[0] / T) / np.exp(dl[0] / T).sum()
    y = 0                                          # q(0) > p(0): accepted with p/q < 1
    ratio = p[y] / q[y]
    assert ratio < 1
    for u, acc in ((ratio * 0.999, True), (ratio * 1.001, False)):
        n, _, _ = fm.verify_sample(tgt[None], dl[None], [[y, 1]], T, np.array([[u, 0.999999]]), 0.5)
        assert (n >= 1) == acc
