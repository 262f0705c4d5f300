"""Prefix trie of a sequence's noise drafts, for target-side tree scoring.

Test infrastructure only (see the package header).

The pages report that drafting several noise samples and scoring them as a
tree adds speed (page "FlashMap并行草拟加速大模型解码", section "6.14 倍是最好成绩…":
a tree of 4 noise drafts, +11 % mean speedup; page "Polymathic AI и
исследователи из Princeton выпустили FlashMap", section "Как FlashMap
показывает себя на бенчмарках?").  Drafts that share a prefix need the
target's distribution after that prefix only once, so the target scores
the unique prefixes -- the nodes of the drafts' prefix trie -- in one pass,
each node attending to the context and to its own ancestors.

Node order (this library's canonical choice; the pages give none):
breadth first -- every node of depth i before any of depth i + 1 -- and,
within a depth, in the order of the first draft whose prefix creates the
node.  Node n stands for a prefix of length depth(n) + 1 ending in
token(n); parent(n) is the node of that prefix without its last token
(-1 at depth 0).  Target row 0 is the root (the empty drafted prefix:
the distribution of the first drafted position); node n's row is 1 + n.
"""
from __future__ import annotations

import math

import numpy as np


def build_trie(drafts):
    """drafts [N][K] tokens -> (token, parent, depth, draft_node [N][K])."""
    drafts = [[int(t) for t in d] for d in drafts]
    N = len(drafts)
    K = len(drafts[0]) if N else 0
    token, parent, depth = [], [], []
    draft_node = [[-1] * K for _ in range(N)]
    for i in range(K):
        seen = {}
        for j in range(N):
            key = (draft_node[j][i - 1] if i > 0 else -1, drafts[j][i])
            if key not in seen:
                seen[key] = len(token)
                token.append(key[1])
                parent.append(key[0])
                depth.append(i)
            draft_node[j][i] = seen[key]
    return token, parent, depth, draft_node


def ancestors(parent):
    """Boolean [n, n]: a[n][m] iff node m is node n or one of its ancestors."""
    n = len(parent)
    a = np.zeros((n, n), dtype=bool)
    for v in range(n):
        u = v
        while u >= 0:
            a[v, u] = True
            u = parent[u]
    return a


def tree_attention(q, k_ctx, v_ctx, k_nodes, v_nodes, parent, n_heads):
    """Attention of every node over [context rows; its ancestors and itself].

    q, k_nodes, v_nodes [n, D]; k_ctx, v_ctx [L, D]; D = n_heads * dh; scale
    1/sqrt(dh).  Returns [n, D].
    """
    q = np.asarray(q, dtype=np.float64)
    n, D = q.shape
    dh = D // n_heads
    anc = ancestors(parent)
    out = np.empty((n, D))
    for v in range(n):
        keys = np.concatenate([k_ctx, k_nodes[anc[v]]], axis=0)
        vals = np.concatenate([v_ctx, v_nodes[anc[v]]], axis=0)
        for h in range(n_heads):
            sl = slice(h * dh, (h + 1) * dh)
            s = keys[:, sl] @ q[v, sl] / math.sqrt(dh)
            w = np.exp(s - s.max())
            out[v, sl] = (w / w.sum()) @ vals[:, sl]
    return out


def draft_rows(node_rows, draft_node):
    """Gather per-draft target rows [N, K+1, ...] from per-node rows
    [1 + n_nodes, ...]: position i of draft j is scored after its first i
    tokens, i.e. by the root row (i = 0) or by node draft_node[j][i-1]."""
    node_rows = np.asarray(node_rows)
    N, K = len(draft_node), len(draft_node[0])
    out = np.empty((N, K + 1) + node_rows.shape[1:], dtype=node_rows.dtype)
    for j in range(N):
        out[j, 0] = node_rows[0]
        for i in range(1, K + 1):
            out[j, i] = node_rows[1 + draft_node[j][i - 1]]
    return out
