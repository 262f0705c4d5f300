"""Two-step draft chain, pinned to a hand-computed fixture.

Fixture ``tests/golden/t6_two_step_zero_dit.txt``: grid 0 -> 0.5 -> 1 of a
zero-DiT drafter with a non-zero time path, sampled at temperature 0.5.  It
fixes what no single-step pin can: the intermediate denoiser
D = softmax(step-1 logits) at temperature 1 (not the sampling temperature),
the move x_1/2 = 1/2 x0 + 1/2 D of the vocabulary-space state, the next
step's embedding x_1/2 . E, and each step's conditioning on its own (s, t).
The flow map with two time points is from page "Polymathic AI и
исследователи из Princeton выпустили FlashMap", section "Как работает
FlashMap?"; two steps trade speed for acceptance (same page, "Как развернуть
FlashMap?").
"""
import math
import os

import numpy as np

from fm_synth import Shape, weight_specs
from oracle import flashmap as fm

GOLD = os.path.join(os.path.dirname(__file__), "golden", "t6_two_step_zero_dit.txt")


def load():
    out = {}
    for line in open(GOLD):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, rest = line.split(None, 1)
        rows = [[float(v) for v in r.split()] for r in rest.split(";")]
        out[key] = np.array(rows) if len(rows) > 1 else np.array(rows[0])
    return out


def model(g):
    s = Shape(V=int(g["V"][0]), d=int(g["d"][0]), n_blocks=int(g["n_blocks"][0]),
              n_heads=int(g["n_heads"][0]), mlp=int(g["mlp"][0]), K=int(g["K"][0]),
              hidden=int(g["hidden"][0]))
    W = {name: np.zeros(shp) for name, shp in weight_specs(s)}
    for k in ("E", "W_lm", "W_ts2", "W_tt2", "W_ada_f"):
        W[k] = g[k].copy()
    for k, name in (("W_ts1_nz", "W_ts1"), ("W_tt1_nz", "W_tt1")):
        r, c, v = g[k]
        W[name][int(r), int(c)] = v
    return s, W


def run(g, temperature):
    s, W = model(g)
    _, kv = fm.project_context(W, s.n_blocks, np.zeros((int(g["ctx"][0]), s.n_taps, s.hidden)))
    u = g["u"][None] if temperature > 0 else None
    return fm.draft(W, s, kv, g["X0"][None], list(g["t_grid"]), temperature, u)


def test_two_step_sampled_matches_hand_values():
    g = load()
    res = run(g, float(g["T"][0]))
    np.testing.assert_allclose(res["step_logits"][0][0], g["logits1"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(res["logits"][0], g["logits2"], rtol=0, atol=1e-13)
    assert res["tokens"][0].tolist() == [int(v) for v in g["tokens_T"]]


def test_two_step_greedy_matches_hand_values():
    g = load()
    res = run(g, 0.0)
    np.testing.assert_allclose(res["logits"][0], g["logits2"], rtol=0, atol=1e-13)
    assert res["tokens"][0].tolist() == [int(v) for v in g["tokens_greedy"]]


# ---- a scalar recomputation of the fixture's chain (math module only) ----
def _silu(a):
    return a / (1.0 + math.exp(-a))


def _g(tau):
    return _silu(_silu(math.cos(1000.0 * tau)))


def _logits(E, W_lm, x, s, t):
    out = []
    for i in range(len(x)):
        z0 = sum(x[i][v] * E[v][0] for v in range(len(E)))
        z1 = sum(x[i][v] * E[v][1] for v in range(len(E)))
        r = ((z0 + math.sin(i)) - (z1 + math.cos(i))) / 2.0
        rho = r / math.sqrt(r * r + 1e-6)
        hf0, hf1 = rho + _g(t), -rho + _g(s)
        out.append([W_lm[v][0] * hf0 + W_lm[v][1] * hf1 for v in range(len(W_lm))])
    return out


def _softmax(row):
    m = max(row)
    e = [math.exp(a - m) for a in row]
    z = sum(e)
    return [a / z for a in e]


def _chain(E, W_lm, X0, t_half=0.5):
    l1 = _logits(E, W_lm, X0, 0.0, t_half)
    D = [_softmax(r) for r in l1]
    a = t_half                                        # (t - s) / (1 - s) at s = 0
    xh = [[X0[i][v] + a * (D[i][v] - X0[i][v]) for v in range(len(E))] for i in range(len(X0))]
    l2 = _logits(E, W_lm, xh, t_half, 1.0)
    return l1, D, xh, l2


def test_fixture_numbers_follow_from_the_scalar_chain():
    g = load()
    l1, D, xh, l2 = _chain(g["E"].tolist(), g["W_lm"].tolist(), g["X0"].tolist())
    for k, v in (("logits1", l1), ("D", D), ("x_half", xh), ("logits2", l2)):
        np.testing.assert_allclose(np.array(v), g[k], rtol=0, atol=1e-15, err_msg=k)
    np.testing.assert_allclose(g["g"], [_g(0.0), _g(0.5), _g(1.0)], rtol=0, atol=1e-16)


def test_two_step_any_noise_matches_scalar_chain():
    # the same zero-DiT model on random noise: the oracle's chain equals the
    # scalar restatement for any state, not only the fixture's
    g = load()
    s, W = model(g)
    _, kv = fm.project_context(W, s.n_blocks, np.zeros((1, s.n_taps, s.hidden)))
    rng = np.random.default_rng(4)
    for _ in range(5):
        X0 = rng.normal(size=(1, s.K, s.V)) * 0.3
        res = fm.draft(W, s, kv, X0, [0.0, 0.5, 1.0])
        l1, _, _, l2 = _chain(W["E"].tolist(), W["W_lm"].tolist(), X0[0].tolist())
        np.testing.assert_allclose(res["step_logits"][0][0], l1, rtol=0, atol=1e-12)
        np.testing.assert_allclose(res["logits"][0], l2, rtol=0, atol=1e-12)
