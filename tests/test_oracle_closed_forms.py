"""Closed forms and invariants that pin the oracle's building blocks.

Each check uses a formula that differs from the oracle's own code path
(an identity, a special case or a textbook value), so a dropped term, a
wrong sign or a swapped operand fails here.
"""
import math

import numpy as np
import pytest
from scipy.special import erf

from oracle import flashmap as fm

RNG = np.random.default_rng(1234)


# ---------------------------------------------------------------- LayerNorm
def test_layer_norm_two_wide_closed_form():
    for a, b in [(3.0, 1.0), (-2.5, 4.0), (1e-4, 0.0)]:
        r = (a - b) / 2
        want = np.array([r, -r]) / math.sqrt(r * r + 1e-6)
        np.testing.assert_allclose(fm.layer_norm0(np.array([a, b])), want, atol=1e-15)


def test_layer_norm_moments():
    x = RNG.normal(3.0, 2.0, size=(7, 129))
    y = fm.layer_norm0(x)
    var = x.var(axis=1)
    np.testing.assert_allclose(y.mean(axis=1), 0, atol=1e-13)
    np.testing.assert_allclose((y * y).mean(axis=1), var / (var + 1e-6), rtol=1e-13)


# ---------------------------------------------------------------- activations
def test_gelu_tanh_identities():
    u = np.linspace(-8, 8, 4001)
    g = fm.gelu_tanh(u)
    # odd part of u * s(u) with s(u) + s(-u) = 1 is exactly u / 2
    np.testing.assert_allclose(g - fm.gelu_tanh(-u), u, atol=1e-13)
    # 0.5 (1 + tanh z) = sigmoid(2 z): an algebraically different form
    z = math.sqrt(2 / math.pi) * (u + 0.044715 * u ** 3)
    np.testing.assert_allclose(g, u / (1 + np.exp(-2 * z)), rtol=1e-12, atol=1e-15)
    # the tanh form tracks the exact erf GELU to < 5e-4 (its published accuracy)
    assert np.abs(g - 0.5 * u * (1 + erf(u / math.sqrt(2)))).max() < 5e-4
    assert fm.gelu_tanh(np.array([0.0]))[0] == 0.0


def test_silu_values():
    assert fm.silu(np.array([0.0]))[0] == 0.0
    u = np.linspace(-6, 6, 101)
    np.testing.assert_allclose(fm.silu(u) - fm.silu(-u), u, atol=1e-14)
    np.testing.assert_allclose(fm.silu(np.array([1.0])), [0.7310585786300049], rtol=1e-15)


def test_softmax_shift_and_temperature():
    z = RNG.normal(size=(3, 50))
    p = fm.softmax(z)
    np.testing.assert_allclose(p.sum(-1), 1, atol=1e-15)
    np.testing.assert_allclose(fm.softmax(z + 7.5), p, atol=1e-15)
    np.testing.assert_allclose(fm.softmax(z, T=2.0), fm.softmax(z / 2.0), atol=1e-15)
    two = fm.softmax(np.array([0.3, -0.4]))
    np.testing.assert_allclose(two[0], 1 / (1 + math.exp(-0.7)), rtol=1e-15)


# ---------------------------------------------------------------- embeddings
def test_time_features_values():
    phi0 = fm.time_features(0.0)
    assert phi0.shape == (256,)
    np.testing.assert_array_equal(phi0, np.r_[np.ones(128), np.zeros(128)])
    tau = math.pi / 2000  # 1000 tau f_0 = pi/2 with f_0 = 1
    phi = fm.time_features(tau)
    assert abs(phi[0]) < 1e-15 and abs(phi[128] - 1) < 1e-15
    # lowest frequency is 1e4^(-127/128)
    f127 = 10000.0 ** (-127 / 128)
    phi = fm.time_features(0.37)
    np.testing.assert_allclose(phi[127], math.cos(370 * f127), rtol=1e-14)
    np.testing.assert_allclose(phi[255], math.sin(370 * f127), rtol=1e-14)
    np.testing.assert_allclose(phi[:128] ** 2 + phi[128:] ** 2, 1, atol=1e-15)


def test_position_embedding_values():
    P = fm.position_embedding(16, 8)
    np.testing.assert_array_equal(P[0], [0, 1, 0, 1, 0, 1, 0, 1])
    np.testing.assert_allclose(P[5, :2], [math.sin(5), math.cos(5)], rtol=1e-15)
    w3 = 10000.0 ** (-6 / 8)
    np.testing.assert_allclose(P[7, 6:8], [math.sin(7 * w3), math.cos(7 * w3)], rtol=1e-14)


# ---------------------------------------------------------------- attention
def _rand_attn(L, K, d):
    return (RNG.normal(size=(K, d)), RNG.normal(size=(L, d)), RNG.normal(size=(L, d)),
            RNG.normal(size=(K, d)), RNG.normal(size=(K, d)))


def test_attention_zero_query_is_mean_of_values():
    Q, Kc, Vc, Kb, Vb = _rand_attn(5, 3, 8)
    O = fm.attention(np.zeros_like(Q), Kc, Vc, Kb, Vb, n_heads=2)
    want = np.concatenate([Vc, Vb]).mean(axis=0)
    np.testing.assert_allclose(O, np.broadcast_to(want, O.shape), atol=1e-14)


def test_attention_single_key_and_two_keys():
    Q, _, _, Kb, Vb = _rand_attn(0, 1, 4)
    empty = np.zeros((0, 4))
    np.testing.assert_allclose(fm.attention(Q, empty, empty, Kb, Vb, 1), Vb, atol=1e-15)
    # two keys: weight of the context key is sigmoid of the scaled score gap
    q = RNG.normal(size=(1, 4)); k1 = RNG.normal(size=(1, 4)); k2 = RNG.normal(size=(1, 4))
    v1 = RNG.normal(size=(1, 4)); v2 = RNG.normal(size=(1, 4))
    gap = float((q @ k1.T - q @ k2.T)[0, 0]) / 2.0   # sqrt(dh) = 2
    w = 1 / (1 + math.exp(-gap))
    np.testing.assert_allclose(fm.attention(q, k1, v1, k2, v2, 1), w * v1 + (1 - w) * v2, atol=1e-14)


def test_attention_heads_are_separate_and_rows_permute():
    Q, Kc, Vc, Kb, Vb = _rand_attn(6, 4, 8)
    O = fm.attention(Q, Kc, Vc, Kb, Vb, n_heads=2)
    Vc2 = Vc.copy(); Vc2[:, 4:] += 10.0
    O2 = fm.attention(Q, Kc, Vc2, Kb, Vb, n_heads=2)
    np.testing.assert_allclose(O2[:, :4], O[:, :4], atol=1e-14)
    perm = RNG.permutation(6)
    np.testing.assert_allclose(fm.attention(Q, Kc[perm], Vc[perm], Kb, Vb, 2), O, atol=1e-13)


# ---------------------------------------------------------------- conditioning
def test_conditioning_wiring():
    # d = 2; embedder s reads phi_0 (cos of the fastest frequency), embedder t
    # reads phi_128 (sin); W2 = I; W_ada = stacked identities.  Then
    # c = [SiLU(phi_0(s)), SiLU(phi_128(t))] and every chunk equals SiLU(c).
    d = 2
    W = {"W_ts1": np.zeros((d, 256)), "W_tt1": np.zeros((d, 256)),
         "W_ts2": np.eye(d), "W_tt2": np.eye(d)}
    W["W_ts1"][0, 0] = 1.0
    W["W_tt1"][1, 128] = 1.0
    W["W_ada.0"] = np.vstack([np.eye(d) * (k + 1) for k in range(6)])
    W["W_ada_f"] = np.vstack([np.eye(d) * -1, np.eye(d) * 3])
    s, t = 0.0, math.pi / 2000
    sig = lambda a: a / (1 + math.exp(-a))
    c = np.array([sig(math.cos(0.0)), sig(math.sin(math.pi / 2))])  # [silu(1), silu(1)]
    sc = np.array([sig(v) for v in c])
    mods, final = fm.conditioning(W, 1, s, t)
    for k in range(6):
        np.testing.assert_allclose(mods[0][k], (k + 1) * sc, rtol=1e-15)
    np.testing.assert_allclose(final[0], -sc, rtol=1e-15)
    np.testing.assert_allclose(final[1], 3 * sc, rtol=1e-15)
    # swapping the roles of s and t changes c (the two times are not symmetric)
    mods2, _ = fm.conditioning(W, 1, t, s)
    assert not np.allclose(mods2[0][0], mods[0][0])


# ---------------------------------------------------------------- one block
def test_block_with_identity_projections():
    # W_q = W_k = 0, W_v = I, W_o = I: attention is uniform, so the first
    # half adds gate1 * mean([V_c; h1]).  W_up = W_down = I: the second half
    # adds gate2 * GELU(h2).  Chunk order is (shift1, scale1, gate1, shift2,
    # scale2, gate2).
    d, K, L = 4, 3, 5
    x = RNG.normal(size=(K, d))
    Vc = RNG.normal(size=(L, d))
    mods = [RNG.normal(size=d) for _ in range(6)]
    sh1, sc1, g1, sh2, sc2, g2 = mods
    W = {"W_qkv.0": np.vstack([np.zeros((2 * d, d)), np.eye(d)]), "W_o.0": np.eye(d),
         "W_up.0": np.eye(d), "W_down.0": np.eye(d)}
    out = fm.dit_block(W, 0, x, mods, np.zeros((L, d)), Vc, n_heads=2)

    def ln(v):
        return (v - v.mean()) / math.sqrt(v.var() + 1e-6)

    h1 = np.array([ln(r) * (1 + sc1) + sh1 for r in x])
    x1 = x + g1 * np.concatenate([Vc, h1]).mean(axis=0)
    h2 = np.array([ln(r) * (1 + sc2) + sh2 for r in x1])
    z = math.sqrt(2 / math.pi) * (h2 + 0.044715 * h2 ** 3)
    want = x1 + g2 * (h2 / (1 + np.exp(-2 * z)))
    np.testing.assert_allclose(out, want, atol=1e-13)


def test_flow_map_update_endpoints():
    x = RNG.normal(size=(2, 5)); D = RNG.normal(size=(2, 5))
    np.testing.assert_allclose(fm.flow_map_update(x, D, 0.0, 1.0), D, atol=1e-15)
    np.testing.assert_allclose(fm.flow_map_update(x, D, 0.5, 1.0), D, atol=1e-15)
    np.testing.assert_allclose(fm.flow_map_update(x, D, 0.0, 0.5), 0.5 * x + 0.5 * D, atol=1e-15)
    np.testing.assert_allclose(fm.flow_map_update(x, D, 0.3, 0.3), x, atol=1e-15)


@pytest.mark.parametrize("u", [0.0, 0.2, 0.5, 0.999999])
def test_inverse_cdf_against_searchsorted(u):
    w = RNG.random(37)
    w[[3, 10]] = 0.0
    got = fm.inverse_cdf(w, u)
    cdf = np.cumsum(w) / w.sum()
    assert got == int(np.searchsorted(cdf, u, side="right"))
    assert w[got] > 0


def test_argmax_ties_lowest():
    assert fm.argmax_lowest(np.array([1.0, 3.0, 3.0, 2.0])) == 1
    assert fm.argmax_lowest(np.zeros(5)) == 0
