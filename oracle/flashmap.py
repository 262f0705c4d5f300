"""Vectorised fp64 oracle: flow-map block draft and prefix verify.

Test infrastructure only (see the package header).  Every function works
in float64 on the exact values the GPU receives (bf16-rounded where the
GPU stores bf16), so rounding of the inputs is not counted as error.

What the pages fix, and what this file takes as the plain reading where
they are silent:

* Speculative round: a drafter proposes K tokens, the target scores them in
  one parallel pass, the longest valid prefix is kept and decoding resumes
  from a target token (P5 "FlashMap Drafts 16 Dependent Tokens at Once",
  section "Why drafting still costs time"; P2 section "Что такое FlashMap?").
  K = 16 (P1 section "一次猜 16 个 token，为什么还会前后不搭").
* The drafter maps Gaussian noise over the vocabulary to a whole block in
  one pass, so one shared noise sample fixes every position jointly (P1 same
  section; P2 section "Почему diffusion-драфтеры теряют в доле принятых
  токенов?").
* The drafter is a DiT of 6 blocks, width 2048, 16 heads, reading the hidden
  states of target layers 1, 9, 17, 25, 33; the embedding matrix and LM head
  come frozen from the target (P1 section "一步生成整块，训练时做了什么";
  P2 section "Как работает FlashMap?").
* The student is a flow map, a denoiser taking two time points, that jumps
  from noise to data (P2 "Как работает FlashMap?"; P1 "一步生成整块…").
  Reading taken: linear interpolant x_t = (1-t) x0 + t x1 between noise x0
  and one-hot data x1; the network outputs D_{s,t} = softmax(logits); the
  map is X_{s,t}(x) = x + ((t-s)/(1-s)) (D_{s,t} - x), so X_{s,1} = D.
* Library choices where the pages say nothing: the noise is soft-embedded
  as x.E; the five hidden states are concatenated and projected by an fc to
  d; each block is adaLN-modulated by the two times; block queries attend
  without a mask over [context rows; block rows]; LayerNorm has no affine
  part and eps 1e-6; GELU uses the tanh form; there are no biases; the
  block slots carry a fixed sin-cos position embedding; the time features
  are the 256-wide sinusoid of 1000*tau; c = TE_s(s) + TE_t(t).
* Lossless verify: greedy keeps the exact-match prefix plus the target's
  argmax; stochastic verify accepts with probability min(1, p/q) and on
  rejection samples the normalised residual max(0, p - q) (P5 "Why drafting
  still costs time"; P1 "能拿来做什么" on probabilistic draft sampling).
"""
from __future__ import annotations

import math

import numpy as np

LN_EPS = 1e-6
TIME_FREQ_DIM = 256
TIME_SCALE = 1000.0


# ---------------------------------------------------------------- elementwise
def layer_norm0(x: np.ndarray) -> np.ndarray:
    """Non-affine LayerNorm over the last axis (population variance, eps 1e-6)."""
    mu = x.mean(axis=-1, keepdims=True)
    xc = x - mu
    var = (xc * xc).mean(axis=-1, keepdims=True)
    return xc / np.sqrt(var + LN_EPS)


def gelu_tanh(u: np.ndarray) -> np.ndarray:
    """GELU, tanh form: u/2 * (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3)))."""
    return 0.5 * u * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (u + 0.044715 * u ** 3)))


def silu(u: np.ndarray) -> np.ndarray:
    return u / (1.0 + np.exp(-u))


def softmax(logits: np.ndarray, T: float = 1.0, axis: int = -1) -> np.ndarray:
    z = np.asarray(logits, dtype=np.float64)
    m = z.max(axis=axis, keepdims=True)
    e = np.exp((z - m) / T)
    return e / e.sum(axis=axis, keepdims=True)


# ---------------------------------------------------------------- embeddings
def time_features(tau: float) -> np.ndarray:
    """256-wide sinusoid of 1000*tau: [cos(1000 tau f_j), sin(1000 tau f_j)], f_j = 1e4^(-j/128)."""
    half = TIME_FREQ_DIM // 2
    f = np.exp(-math.log(10000.0) * np.arange(half, dtype=np.float64) / half)
    a = TIME_SCALE * float(tau) * f
    return np.concatenate([np.cos(a), np.sin(a)])


def position_embedding(K: int, d: int) -> np.ndarray:
    """Fixed sin-cos embedding of block slot i: P[i,2k]=sin(i w_k), P[i,2k+1]=cos(i w_k), w_k=1e4^(-2k/d)."""
    P = np.zeros((K, d), dtype=np.float64)
    i = np.arange(K, dtype=np.float64)[:, None]
    w = 10000.0 ** (-2.0 * np.arange(d // 2, dtype=np.float64) / d)
    P[:, 0::2] = np.sin(i * w)
    P[:, 1::2] = np.cos(i * w)
    return P


def _f64(W: dict) -> dict:
    return {k: np.asarray(v, dtype=np.float64) for k, v in W.items()}


# ---------------------------------------------------------------- conditioning
def conditioning(W: dict, n_blocks: int, s: float, t: float):
    """adaLN modulation for the step s -> t.

    c = TE_s(s) + TE_t(t), TE(tau) = W2 SiLU(W1 phi(tau)).  Block l gets
    (shift1, scale1, gate1, shift2, scale2, gate2) = split6(W_ada,l SiLU(c));
    the final norm gets (shift_f, scale_f) = split2(W_ada,f SiLU(c)).
    """
    te_s = W["W_ts2"] @ silu(W["W_ts1"] @ time_features(s))
    te_t = W["W_tt2"] @ silu(W["W_tt1"] @ time_features(t))
    sc = silu(te_s + te_t)
    mods = []
    for l in range(n_blocks):
        m = W[f"W_ada.{l}"] @ sc
        mods.append(np.split(m, 6))
    final = np.split(W["W_ada_f"] @ sc, 2)
    return mods, final


# ---------------------------------------------------------------- context
def project_context(W: dict, n_blocks: int, hidden: np.ndarray):
    """Context features and per-block keys/values.

    hidden [L, n_taps, H] -> C = LN0(concat_taps(hidden) W_fc^T) [L, d];
    block l: K_c = C W_k,l^T, V_c = C W_v,l^T with W_k, W_v the key and value
    thirds of W_qkv,l (the same projections the block rows use).
    """
    L = hidden.shape[0]
    flat = np.asarray(hidden, dtype=np.float64).reshape(L, hidden.shape[1] * hidden.shape[2])
    C = layer_norm0(flat @ W["W_fc"].T)
    d = C.shape[1]
    kv = []
    for l in range(n_blocks):
        Wqkv = W[f"W_qkv.{l}"]
        kv.append((C @ Wqkv[d:2 * d].T, C @ Wqkv[2 * d:].T))
    return C, kv


# ---------------------------------------------------------------- DiT
def attention(Q, Kc, Vc, Kb, Vb, n_heads):
    """Unmasked attention of the block rows over [context rows; block rows], per head."""
    K, d = Q.shape
    dh = d // n_heads
    keys = np.concatenate([Kc, Kb], axis=0)
    vals = np.concatenate([Vc, Vb], axis=0)
    O = np.empty_like(Q)
    for h in range(n_heads):
        sl = slice(h * dh, (h + 1) * dh)
        S = Q[:, sl] @ keys[:, sl].T / math.sqrt(dh)
        O[:, sl] = softmax(S, axis=-1) @ vals[:, sl]
    return O


def dit_block(W, l, x, mods_l, Kc, Vc, n_heads):
    """One adaLN DiT block on the rows of one noise draft (x: [K, d])."""
    d = x.shape[1]
    sh1, sc1, g1, sh2, sc2, g2 = mods_l
    h = layer_norm0(x) * (1.0 + sc1) + sh1
    qkv = h @ W[f"W_qkv.{l}"].T
    Q, Kb, Vb = qkv[:, :d], qkv[:, d:2 * d], qkv[:, 2 * d:]
    O = attention(Q, Kc, Vc, Kb, Vb, n_heads)
    x = x + g1 * (O @ W[f"W_o.{l}"].T)
    h = layer_norm0(x) * (1.0 + sc2) + sh2
    x = x + g2 * (gelu_tanh(h @ W[f"W_up.{l}"].T) @ W[f"W_down.{l}"].T)
    return x


def dit_logits(W, shape, z, ctx_kv, mods, final):
    """Logits [N, K, V] of the DiT applied to embedded blocks z [N, K, d]."""
    N, K, d = z.shape
    P = position_embedding(K, d)
    out = np.empty((N, K, shape.V))
    for j in range(N):
        x = z[j] + P
        for l in range(shape.n_blocks):
            x = dit_block(W, l, x, mods[l], ctx_kv[l][0], ctx_kv[l][1], shape.n_heads)
        shf, scf = final
        hf = layer_norm0(x) * (1.0 + scf) + shf
        out[j] = hf @ W["W_lm"].T
    return out


def flow_map_update(x: np.ndarray, D: np.ndarray, s: float, t: float) -> np.ndarray:
    """X_{s,t}(x) = x + ((t - s)/(1 - s)) (D - x); equals D at t = 1."""
    return x + ((t - s) / (1.0 - s)) * (D - x)


# ---------------------------------------------------------------- token choice
def argmax_lowest(row: np.ndarray) -> int:
    """Index of the largest entry; ties go to the lowest index.

    NaN entries never win: they rank below every number, -inf included.  A
    row with no entry other than NaN gives index 0.
    """
    row = np.asarray(row)
    ok = np.flatnonzero(~np.isnan(row))
    if ok.size == 0:
        return 0
    return int(ok[np.argmax(row[ok])])


def inverse_cdf(weights: np.ndarray, u: float) -> int:
    """Smallest v whose running sum (vocab order) exceeds u * total.

    If rounding leaves no such v, the last v with positive weight.
    """
    c = np.cumsum(weights)
    idx = np.nonzero(c > u * c[-1])[0]
    if idx.size:
        return int(idx[0])
    return int(np.nonzero(weights > 0)[0][-1])


def sample_row(logits: np.ndarray, T: float, u: float) -> int:
    """Token drawn from softmax(logits / T) by inverse CDF at u."""
    z = np.asarray(logits, dtype=np.float64)
    return inverse_cdf(np.exp((z - z.max()) / T), u)


# ---------------------------------------------------------------- draft
def draft(W, shape, ctx_kv, X0, t_grid, temperature=0.0, u_draft=None):
    """Draft one sequence's noise blocks X0 [N, K, V] along the time grid.

    Returns dict(tokens [N, K], logits [N, K, V] of the last step,
    step_logits list).  Each step embeds the current vocab-space state,
    z = x_s E, runs the DiT conditioned on (s, t) and, for t < 1, moves the
    state by the flow-map update with D = softmax(logits) at temperature 1.
    At t = 1 tokens are the argmax (temperature 0) or an inverse-CDF draw
    from softmax(logits / T) at the host-supplied uniforms.
    """
    x = np.asarray(X0, dtype=np.float64)
    grid = [float(v) for v in t_grid]
    assert grid[0] == 0.0 and grid[-1] == 1.0 and all(a < b for a, b in zip(grid, grid[1:]))
    step_logits = []
    logits = None
    for s, t in zip(grid[:-1], grid[1:]):
        mods, final = conditioning(W, shape.n_blocks, s, t)
        z = x @ W["E"]
        logits = dit_logits(W, shape, z, ctx_kv, mods, final)
        step_logits.append(logits)
        if t < 1.0:
            x = flow_map_update(x, softmax(logits, 1.0), s, t)
    N, K, _ = logits.shape
    tokens = np.empty((N, K), dtype=np.int64)
    for j in range(N):
        for i in range(K):
            if temperature == 0.0:
                tokens[j, i] = argmax_lowest(logits[j, i])
            else:
                tokens[j, i] = sample_row(logits[j, i], temperature, float(u_draft[j, i]))
    return {"tokens": tokens, "logits": logits, "step_logits": step_logits}


def margins(logits: np.ndarray) -> np.ndarray:
    """Top-1 minus top-2 logit per row."""
    part = np.partition(np.asarray(logits, dtype=np.float64), -2, axis=-1)
    return part[..., -1] - part[..., -2]


# ---------------------------------------------------------------- verify
def verify_greedy(target, draft_tokens):
    """Greedy verify of N drafts of one sequence.

    target [N, K+1, V]: row i of draft j scores position i+1 after that
    draft's first i tokens.  Per draft, n_j counts the leading drafted
    tokens equal to the target argmax.  The branch is the draft with the
    largest n_j (lowest index on ties); the output is its first n tokens
    followed by the target argmax at position n+1.
    """
    target = np.asarray(target)
    N, K1, V = target.shape
    K = K1 - 1
    best_n, best_j = -1, 0
    for j in range(N):
        n = 0
        while n < K and int(draft_tokens[j][n]) == argmax_lowest(target[j, n]):
            n += 1
        if n > best_n:
            best_n, best_j = n, j
    out = [int(draft_tokens[best_j][i]) for i in range(best_n)]
    out.append(argmax_lowest(target[best_j, best_n]))
    return best_n, best_j, out


def _probs(row, T):
    z = np.asarray(row, dtype=np.float64)
    e = np.exp((z - z.max()) / T)
    return e / e.sum()


def verify_sample(target, draft_logits, draft_tokens, T, u_accept, u_res):
    """Stochastic verify of N drafts (N = 1: plain speculative sampling).

    p = softmax(target / T) on the rows of the accepted prefix; q^j =
    softmax(draft_logits^j / T), or the point mass on the drafted token when
    ``draft_logits`` is None (greedy draft).  At depth i the alive drafts
    (those whose first i-1 tokens equal the accepted prefix) are tried in
    index order: draft j is accepted iff u_accept[j, i] * q^j_i(y) < p'(y);
    otherwise p' becomes normalise(max(0, p' - q^j_i)) and the next alive
    draft is tried.  If none is accepted, one token is drawn from p' by
    inverse CDF at u_res and the round ends.  If all K depths accept, the
    bonus token is drawn from the accepted branch's row K+1 at u_res.

    Returns (n accepted, branch, tokens): branch is the lowest-index draft
    whose tokens equal the accepted prefix.
    """
    target = np.asarray(target)
    N, K1, V = target.shape
    K = K1 - 1
    alive = list(range(N))
    out = []
    for i in range(K):
        pp = _probs(target[alive[0], i], T)
        accepted = None
        for j in alive:
            y = int(draft_tokens[j][i])
            if draft_logits is None:
                q = np.zeros(V)
                q[y] = 1.0
            else:
                q = _probs(draft_logits[j][i], T)
            if float(u_accept[j][i]) * q[y] < pp[y]:
                accepted = y
                break
            r = np.maximum(pp - q, 0.0)
            z = r.sum()
            if z > 0.0:
                pp = r / z
        if accepted is None:
            out.append(inverse_cdf(pp, float(u_res)))
            return i, alive[0], out
        out.append(accepted)
        alive = [j for j in alive if int(draft_tokens[j][i]) == accepted]
    out.append(inverse_cdf(_probs(target[alive[0], K], T), float(u_res)))
    return K, alive[0], out
