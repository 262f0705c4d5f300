"""Two independent CPU formulations of the draft agree (vectorised vs loops)."""
import dataclasses

import numpy as np
import pytest

import fm_synth as fs
from oracle import flashmap as fm
from oracle import loops


def _case(shape, seed_round=0, ctx=6):
    w = dataclasses.replace(fs.WORKLOADS["tiny_f32"], shape=shape, ctx=ctx)
    W = fs.make_weights(shape, "f32", std=0.02)
    W = {k: v * 5.0 for k, v in W.items()}   # larger weights: non-trivial gates
    hid = fs.prefill_hidden(w, 0)
    ri = fs.round_inputs(w, seed_round)
    return W, hid, ri.noise[0, 0]


@pytest.mark.parametrize("s,t", [(0.0, 1.0), (0.5, 1.0)])
def test_loops_match_vectorised(s, t):
    shape = fs.Shape(V=64, d=32, n_blocks=2, n_heads=4, mlp=48, K=5, hidden=8)
    W, hid, X0 = _case(shape)
    Wd = {k: np.asarray(v, dtype=np.float64) for k, v in W.items()}
    _, kv = fm.project_context(Wd, shape.n_blocks, hid)
    mods, final = fm.conditioning(Wd, shape.n_blocks, s, t)
    want = fm.dit_logits(Wd, shape, (X0.astype(np.float64) @ Wd["E"])[None], kv, mods, final)[0]
    got, tok = loops.draft_tokens_loops(W, shape, hid, X0, s=s, t=t)
    got = np.array(got)
    scale = np.abs(want).max()
    assert np.abs(got - want).max() <= 1e-12 * scale
    assert tok == [fm.argmax_lowest(r) for r in want]
    # the update really changes things: gates are far from zero at this scale
    assert np.abs(mods[0][2]).max() > 0.05


def test_loops_match_vectorised_tiny_config():
    w = fs.WORKLOADS["tiny_f32"]
    shape = w.shape
    W = fs.make_weights(shape, "f32")
    Wd = {k: np.asarray(v, dtype=np.float64) for k, v in W.items()}
    hid = fs.prefill_hidden(w, 0)
    X0 = fs.round_inputs(w, 0).noise[0, 0]
    _, kv = fm.project_context(Wd, shape.n_blocks, hid)
    res = fm.draft(Wd, shape, kv, X0[None], w.t_grid)
    got, tok = loops.draft_tokens_loops(W, shape, hid, X0)
    want = res["logits"][0]
    assert np.abs(np.array(got) - want).max() <= 1e-12 * np.abs(want).max()
    assert tok == res["tokens"][0].tolist()
