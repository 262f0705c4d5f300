"""Plain-loop fp64 draft for tiny shapes: a second, independent formulation.

Test infrastructure only.  Written with Python lists, ``math`` and explicit
loops from the same definitions as ``oracle.flashmap`` (see that module's
header for the pages' passages and the readings taken), without importing
it, so that an indexing or transposition slip in one formulation shows up
as a disagreement between the two.  Intended for V, d <= a few hundred.
"""
from __future__ import annotations

import math
from operator import mul

EPS = 1e-6


def _dot(a, b):
    return math.fsum(map(mul, a, b))


def _matvec(rows, x):
    """rows: list of output rows [out][in]; returns [out]."""
    return [_dot(r, x) for r in rows]


def _ln0(v):
    n = len(v)
    mu = math.fsum(v) / n
    c = [a - mu for a in v]
    var = math.fsum(a * a for a in c) / n
    s = 1.0 / math.sqrt(var + EPS)
    return [a * s for a in c]


def _silu(a):
    return a / (1.0 + math.exp(-a))


def _gelu(a):
    return 0.5 * a * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * (a + 0.044715 * a * a * a)))


def _rows(M):
    return [[float(v) for v in r] for r in M]


def _phi(tau):
    out_c, out_s = [], []
    for j in range(128):
        f = 10000.0 ** (-j / 128.0)
        out_c.append(math.cos(1000.0 * tau * f))
        out_s.append(math.sin(1000.0 * tau * f))
    return out_c + out_s


def draft_tokens_loops(W, shape, hidden, X0, s=0.0, t=1.0):
    """One-step greedy draft of a single block with plain loops.

    W: dict of weights (array-likes), shape: fm_synth.Shape, hidden
    [L][n_taps][H] context states, X0 [K][V] noise.  Returns (logits [K][V],
    tokens [K]).
    """
    d, V, K, nb, nh = shape.d, shape.V, shape.K, shape.n_blocks, shape.n_heads
    dh = d // nh

    # conditioning: two time embedders, summed, through SiLU
    def te(w1, w2, tau):
        return _matvec(_rows(w2), [_silu(a) for a in _matvec(_rows(w1), _phi(tau))])

    c = [a + b for a, b in zip(te(W["W_ts1"], W["W_ts2"], s), te(W["W_tt1"], W["W_tt2"], t))]
    sc = [_silu(a) for a in c]
    mods = []
    for l in range(nb):
        m = _matvec(_rows(W[f"W_ada.{l}"]), sc)
        mods.append([m[k * d:(k + 1) * d] for k in range(6)])
    mf = _matvec(_rows(W["W_ada_f"]), sc)
    shf, scf = mf[:d], mf[d:]

    # context features: fc over the concatenated taps, then LN0
    Wfc = _rows(W["W_fc"])
    C = []
    for row in hidden:
        flat = [float(v) for tap in row for v in tap]
        C.append(_ln0(_matvec(Wfc, flat)))

    # input embedding: z = x0 . E plus slot position
    E = _rows(W["E"])
    x = []
    for i in range(K):
        xi = [float(v) for v in X0[i]]
        z = [0.0] * d
        for c_ in range(d):
            z[c_] = math.fsum(xi[v] * E[v][c_] for v in range(V))
        for k in range(d // 2):
            w = 10000.0 ** (-2.0 * k / d)
            z[2 * k] += math.sin(i * w)
            z[2 * k + 1] += math.cos(i * w)
        x.append(z)

    for l in range(nb):
        sh1, sc1, g1, sh2, sc2, g2 = mods[l]
        Wqkv = _rows(W[f"W_qkv.{l}"])
        Wq, Wk, Wv = Wqkv[:d], Wqkv[d:2 * d], Wqkv[2 * d:]
        Kc = [_matvec(Wk, crow) for crow in C]
        Vc = [_matvec(Wv, crow) for crow in C]
        h = [[a * (1.0 + b) + e for a, b, e in zip(_ln0(xi), sc1, sh1)] for xi in x]
        Q = [_matvec(Wq, hi) for hi in h]
        Kb = [_matvec(Wk, hi) for hi in h]
        Vb = [_matvec(Wv, hi) for hi in h]
        keys, vals = Kc + Kb, Vc + Vb
        O = [[0.0] * d for _ in range(K)]
        for hd in range(nh):
            lo = hd * dh
            for i in range(K):
                sc_ = [_dot(Q[i][lo:lo + dh], kk[lo:lo + dh]) / math.sqrt(dh) for kk in keys]
                m = max(sc_)
                e = [math.exp(a - m) for a in sc_]
                Z = math.fsum(e)
                for c_ in range(dh):
                    O[i][lo + c_] = math.fsum(e[r] * vals[r][lo + c_] for r in range(len(keys))) / Z
        Wo = _rows(W[f"W_o.{l}"])
        for i in range(K):
            y = _matvec(Wo, O[i])
            x[i] = [a + g * b for a, g, b in zip(x[i], g1, y)]
        W1 = _rows(W[f"W_up.{l}"])
        W2 = _rows(W[f"W_down.{l}"])
        for i in range(K):
            hi = [a * (1.0 + b) + e for a, b, e in zip(_ln0(x[i]), sc2, sh2)]
            u = [_gelu(a) for a in _matvec(W1, hi)]
            y = _matvec(W2, u)
            x[i] = [a + g * b for a, g, b in zip(x[i], g2, y)]

    Wlm = _rows(W["W_lm"])
    logits, tokens = [], []
    for i in range(K):
        hf = [a * (1.0 + b) + e for a, b, e in zip(_ln0(x[i]), scf, shf)]
        row = _matvec(Wlm, hf)
        logits.append(row)
        best = 0
        for v in range(1, V):
            if row[v] > row[best]:
                best = v
        tokens.append(best)
    return logits, tokens
