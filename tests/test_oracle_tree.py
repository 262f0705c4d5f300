"""Prefix trie and tree attention of the oracle, pinned without the oracle.

The trie groups drafts that share a prefix (page "FlashMap并行草拟加速大模型解码",
section "6.14 倍是最好成绩…": a tree of 4 noise drafts).  Pins: a hand-built
fixture; brute-force prefix equality on random drafts; and tree attention
against plain causal attention along each draft's own path (the textbook
definition the tree must reproduce for every node).
"""
import math
import os

import numpy as np
import pytest

from oracle import tree as ot

GOLD = os.path.join(os.path.dirname(__file__), "golden", "t7_tree_of_four_drafts.txt")


def _load():
    out = {}
    for line in open(GOLD):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, rest = line.split(None, 1)
        out[key] = [[int(v) for v in r.split()] for r in rest.split(";")]
    return out


def test_hand_built_trie():
    g = _load()
    token, parent, depth, dn = ot.build_trie(g["drafts"])
    assert token == g["token"][0] and parent == g["parent"][0] and depth == g["depth"][0]
    assert dn == g["draft_node"]
    rows = ot.draft_rows(np.arange(1 + len(token)), dn)
    assert rows[1].tolist() == g["rows_of_draft_1"][0]


def _random_drafts(rng, N, K, V):
    d = rng.integers(0, V, size=(N, K))
    for j in range(1, N):
        cut = int(rng.integers(0, K + 1))
        src = int(rng.integers(0, j))
        d[j, :cut] = d[src, :cut]
    return d


@pytest.mark.parametrize("seed", range(6))
def test_trie_matches_brute_force_prefixes(seed):
    rng = np.random.default_rng(seed)
    N, K, V = int(rng.integers(1, 6)), int(rng.integers(1, 7)), int(rng.integers(2, 5))
    d = _random_drafts(rng, N, K, V)
    token, parent, depth, dn = ot.build_trie(d)
    prefixes = {tuple(d[j, :i + 1]) for j in range(N) for i in range(K)}
    assert len(token) == len(prefixes)
    for j in range(N):
        for i in range(K):
            n = dn[j][i]
            assert token[n] == d[j, i] and depth[n] == i
            assert parent[n] == (dn[j][i - 1] if i else -1)
            for j2 in range(N):
                same = tuple(d[j, :i + 1]) == tuple(d[j2, :i + 1])
                assert (dn[j2][i] == n) == same
    # breadth first, parents first
    assert depth == sorted(depth)
    assert all(p < v for v, p in enumerate(parent))


def test_tree_attention_equals_causal_attention_on_each_path():
    rng = np.random.default_rng(7)
    N, K, V, H, dh, L = 4, 5, 3, 2, 8, 6
    d = _random_drafts(rng, N, K, V)
    token, parent, depth, dn = ot.build_trie(d)
    n = len(token)
    D = H * dh
    q, kn, vn = (rng.normal(size=(n, D)) for _ in range(3))
    kc, vc = rng.normal(size=(L, D)), rng.normal(size=(L, D))
    got = ot.tree_attention(q, kc, vc, kn, vn, parent, H)
    for j in range(N):
        path = [dn[j][i] for i in range(K)]
        for i in range(K):
            # plain causal attention of draft j's position i over the context
            # and the draft's own positions 0..i
            keys = np.concatenate([kc, kn[path[:i + 1]]])
            vals = np.concatenate([vc, vn[path[:i + 1]]])
            for h in range(H):
                sl = slice(h * dh, (h + 1) * dh)
                s = np.array([sum(q[path[i], c] * keys[r, c] for c in range(h * dh, (h + 1) * dh))
                              for r in range(len(keys))]) / math.sqrt(dh)
                w = [math.exp(x - max(s)) for x in s]
                want = sum(w[r] * vals[r, sl] for r in range(len(keys))) / sum(w)
                np.testing.assert_allclose(got[path[i], sl], want, rtol=0, atol=1e-12)


def test_ancestor_sets():
    g = _load()
    _, parent, _, _ = ot.build_trie(g["drafts"])
    a = ot.ancestors(parent)
    assert set(np.flatnonzero(a[5])) == {0, 2, 5}
    assert set(np.flatnonzero(a[8])) == {1, 4, 8}
    assert a.sum() == sum(dep + 1 for dep in g["depth"][0])
