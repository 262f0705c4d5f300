"""Hand-computed zero-DiT draft (fixture tests/golden/t1_zero_dit_draft.txt).

Pins the oracle's soft embedding, slot position embedding, final LN0, LM
head, argmax tie-break and greedy verify to values derived by hand.
"""
import math
import os

import numpy as np

from fm_synth import Shape, weight_specs
from oracle import flashmap as fm

GOLD = os.path.join(os.path.dirname(__file__), "golden", "t1_zero_dit_draft.txt")


def _load():
    out = {}
    for line in open(GOLD):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, rest = line.split(None, 1)
        rows = [[float(v) for v in r.split()] for r in rest.split(";")]
        out[key] = np.array(rows) if len(rows) > 1 else np.array(rows[0])
    return out


def _zero_model(g):
    s = Shape(V=int(g["V"][0]), d=int(g["d"][0]), n_blocks=int(g["n_blocks"][0]),
              n_heads=int(g["n_heads"][0]), mlp=int(g["mlp"][0]), K=int(g["K"][0]),
              hidden=int(g["hidden"][0]))
    W = {name: np.zeros(shp) for name, shp in weight_specs(s)}
    W["E"] = g["E"]
    W["W_lm"] = g["W_lm"]
    return s, W


def test_zero_dit_draft_matches_hand_values():
    g = _load()
    s, W = _zero_model(g)
    hidden = np.ones((int(g["ctx"][0]), s.n_taps, s.hidden))
    _, kv = fm.project_context(W, s.n_blocks, hidden)
    res = fm.draft(W, s, kv, g["X0"][None], [0.0, 1.0], temperature=0.0)
    assert res["tokens"][0].tolist() == [int(v) for v in g["expected_tokens"]]
    np.testing.assert_allclose(res["logits"][0], g["expected_logits"], rtol=0, atol=1e-15)


def test_zero_dit_closed_form_any_noise():
    # For any noise row, the zero-DiT logits are sign(a-b)-scaled differences
    # of the LM-head columns: logits_v = rho(r) * (W_lm[v,0] - W_lm[v,1]).
    g = _load()
    s, W = _zero_model(g)
    rng = np.random.default_rng(0)
    X0 = rng.normal(size=(1, s.K, s.V))
    _, kv = fm.project_context(W, s.n_blocks, np.zeros((1, s.n_taps, s.hidden)))
    res = fm.draft(W, s, kv, X0, [0.0, 1.0])
    for i in range(s.K):
        z0 = sum(X0[0, i, v] * W["E"][v, 0] for v in range(s.V)) + math.sin(i)
        z1 = sum(X0[0, i, v] * W["E"][v, 1] for v in range(s.V)) + math.cos(i)
        r = (z0 - z1) / 2
        rho = r / math.sqrt(r * r + 1e-6)
        want = [rho * (W["W_lm"][v, 0] - W["W_lm"][v, 1]) for v in range(s.V)]
        np.testing.assert_allclose(res["logits"][0, i], want, rtol=0, atol=1e-13)


def test_hand_greedy_verify():
    g = _load()
    n, branch, out = fm.verify_greedy(g["target"][None], [[int(v) for v in g["expected_tokens"]]])
    assert n == int(g["expected_n"][0]) and branch == 0
    assert out == [int(v) for v in g["expected_out"]]
