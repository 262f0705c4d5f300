"""Verify is lossless: exact enumeration of the output distribution.

The pages define a lossless verifier as one that keeps the target model's
output distribution under the same sampling settings, and greedy
speculative output as equal to plain greedy target decoding (page "FlashMap
Drafts 16 Dependent Tokens at Once…", section "Why drafting still costs
time"; page "FlashMap并行草拟加速大模型解码", section "一次猜 16 个 token，为什么还会前后不搭").

The oracle's stochastic verify is a deterministic function of host-supplied
uniforms, piecewise constant in each of them.  The enumeration below walks
every cell: whenever the oracle reads a uniform that is not yet fixed, the
walk branches over the cells cut by every threshold that uniform could be
compared with (acceptance ratios min(1, p/q) and CDF breakpoints of every
reachable residual), evaluates the oracle at each cell's midpoint and
weights the branch by the cell's width.  Each output is extended to K+1
tokens with the exact target conditionals; the resulting distribution must
equal the target's own product distribution.
"""
import itertools

import numpy as np
import pytest

from oracle import flashmap as fm


class _Unset(Exception):
    def __init__(self, key):
        self.key = key


class _LazyU:
    def __init__(self, assign, key):
        self.assign, self.key = assign, key

    def __float__(self):
        if self.key not in self.assign:
            raise _Unset(self.key)
        return self.assign[self.key]


class _LazyRows:
    def __init__(self, assign, N, K):
        self.rows = [[_LazyU(assign, ("a", j, i)) for i in range(K)] for j in range(N)]

    def __getitem__(self, j):
        return self.rows[j]


def _cells(points):
    pts = sorted({0.0, 1.0, *[min(1.0, max(0.0, float(p))) for p in points]})
    return [(a, b) for a, b in zip(pts, pts[1:]) if b > a]


def _residual(p, q):
    r = np.maximum(p - q, 0.0)
    z = r.sum()
    return r / z if z > 0 else p


def _enumerate(run, breakpoints):
    """Sum weight over all cells; run(assign) returns an outcome or raises _Unset."""
    out = {}
    stack = [({}, 1.0)]
    while stack:
        assign, w = stack.pop()
        try:
            res = run(assign)
        except _Unset as e:
            for a, b in _cells(breakpoints(e.key)):
                nxt = dict(assign)
                nxt[e.key] = 0.5 * (a + b)
                stack.append((nxt, w * (b - a)))
            continue
        out[res] = out.get(res, 0.0) + w
    return out


def _target_table(rng, V, K):
    """p(. | prefix) for every prefix of length 0..K, as a dict."""
    table = {}
    for L in range(K + 1):
        for pre in itertools.product(range(V), repeat=L):
            p = rng.random(V) + 0.05
            table[pre] = p / p.sum()
    return table


def _check_lossless(V, K, N, seed, greedy_draft=False, T=1.0):
    """Exact output distribution of the oracle's stochastic verify at
    temperature T.  Logits are T * log(probabilities), so softmax(logits / T)
    is the intended distribution: a verify that multiplies by T where it should
    divide (or ignores T) breaks the equality unless T = 1."""
    rng = np.random.default_rng(seed)
    table = _target_table(rng, V, K)
    qs = []
    for j in range(N):
        q = rng.random((K, V)) + 0.05
        qs.append(q / q.sum(axis=1, keepdims=True))
    full = {}
    drafts = itertools.product(*[itertools.product(range(V), repeat=K) for _ in range(N)])
    if greedy_draft:
        drafts = [tuple(tuple(int(np.argmax(qs[j][i])) for i in range(K)) for j in range(N))]
    for ys in drafts:
        pq = 1.0 if greedy_draft else float(np.prod([qs[j][i][ys[j][i]] for j in range(N) for i in range(K)]))
        target = T * np.array([[np.log(table[ys[j][:i]]) for i in range(K + 1)] for j in range(N)])
        dlog = None if greedy_draft else T * np.array([np.log(qs[j]) for j in range(N)])
        qd = [[(np.eye(V)[ys[j][i]] if greedy_draft else qs[j][i]) for i in range(K)] for j in range(N)]

        # every distribution any uniform can be compared against
        cands = {}
        for i in range(K + 1):
            rows = {ys[j][:i] for j in range(N)}
            for pre in rows:
                dists = [table[pre]]
                if i < K:
                    for order in itertools.permutations(range(N)):
                        for m in range(1, N + 1):
                            p = table[pre]
                            for j in order[:m]:
                                p = _residual(p, qd[j][i])
                            dists.append(p)
                cands.setdefault(i, []).extend(dists)

        def bps(key):
            if key[0] == "a":
                _, j, i = key
                y = ys[j][i]
                return [p[y] / qd[j][i][y] for p in cands[i]]
            pts = []
            for ds in cands.values():
                for p in ds:
                    pts.extend(np.cumsum(p)[:-1] / p.sum())
            return pts

        def run(assign):
            ua = _LazyRows(assign, N, K)
            ur = _LazyU(assign, ("r",))
            n, branch, toks = fm.verify_sample(target, dlog, ys, T, ua, ur)
            return tuple(toks)

        for toks, w in _enumerate(run, bps).items():
            # extend to K+1 tokens with exact target conditionals
            L = len(toks)
            for tail in itertools.product(range(V), repeat=K + 1 - L):
                seq = toks + tail
                pr = w * pq
                for i in range(L, K + 1):
                    pr *= table[seq[:i]][seq[i]]
                full[seq] = full.get(seq, 0.0) + pr
    for seq in itertools.product(range(V), repeat=K + 1):
        want = np.prod([table[seq[:i]][seq[i]] for i in range(K + 1)])
        assert abs(full.get(seq, 0.0) - want) < 1e-12, (seq, full.get(seq), want)
    assert abs(sum(full.values()) - 1.0) < 1e-12


def test_lossless_single_draft_V6_K3():
    _check_lossless(V=6, K=3, N=1, seed=11)


def test_lossless_tree_two_drafts_V4_K2():
    _check_lossless(V=4, K=2, N=2, seed=12)


def test_lossless_greedy_draft_stochastic_verify():
    _check_lossless(V=5, K=3, N=1, seed=13, greedy_draft=True)


# Temperature other than 1: the target and draft distributions are
# softmax(logits / T) (page "FlashMap并行草拟加速大模型解码", section "能拿来做什么":
# probabilistic draft sampling at T > 0; lossless at the same sampling settings,
# page "FlashMap Drafts 16 Dependent Tokens at Once…", "Why drafting still costs time").
@pytest.mark.parametrize("T", [2.0, 0.5])
def test_lossless_single_draft_V5_K2_temperature(T):
    _check_lossless(V=5, K=2, N=1, seed=14, T=T)


def test_lossless_tree_two_drafts_V4_K2_T2():
    _check_lossless(V=4, K=2, N=2, seed=12, T=2.0)


def test_lossless_greedy_draft_T2():
    _check_lossless(V=5, K=3, N=1, seed=13, greedy_draft=True, T=2.0)


def test_accept_probabilities():
    rng = np.random.default_rng(5)
    V, K = 7, 4
    p = rng.random((K + 1, V)); p /= p.sum(1, keepdims=True)
    # p == q: every position is accepted whatever the uniforms
    for _ in range(50):
        y = [int(rng.integers(V)) for _ in range(K)]
        n, _, toks = fm.verify_sample(np.log(p)[None], np.log(p[:K])[None], [y], 1.0,
                                      rng.random((1, K)), rng.random())
        assert n == K and toks[:K] == y
    # q = point mass on y: position 1 is accepted iff u < p(y)
    y = [3] * K
    for u in [0.0, p[0, 3] * 0.999, p[0, 3] * 1.001, 0.99]:
        ua = np.full((1, K), 0.999999)
        ua[0, 0] = u
        n, _, toks = fm.verify_sample(np.log(p)[None], None, [y], 1.0, ua, 0.5)
        assert (n >= 1) == (u < p[0, 3])
        if n == 0:
            assert toks[0] != 3   # the residual excludes the rejected token


def test_greedy_verify_tree_branch_rules():
    V, K = 5, 3
    rng = np.random.default_rng(3)
    t = rng.normal(size=(2, K + 1, V))
    a = t.argmax(-1)
    d0 = [a[0, 0], (a[0, 1] + 1) % V, 0]              # n = 1
    d1 = [a[1, 0], a[1, 1], (a[1, 2] + 1) % V]        # n = 2
    n, b, out = fm.verify_greedy(t, [d0, d1])
    assert (n, b) == (2, 1) and out == [int(a[1, 0]), int(a[1, 1]), int(a[1, 2])]
    # ties in n go to the lowest draft index
    n, b, _ = fm.verify_greedy(t[[1, 1]], [d1, d1])
    assert (n, b) == (2, 0)
    # a single draft is plain greedy verify
    n1, _, out1 = fm.verify_greedy(t[:1], [d0])
    assert n1 == 1 and out1 == [int(a[0, 0]), int(a[0, 1])]
