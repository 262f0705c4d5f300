"""Flow-map drafting on the exact two-mode toy ("new york" / "san diego").

Pins the oracle's flow-map update and its joint (shared-noise) token choice
against an exact flow: one noise sample mapped to a whole block never mixes
the modes, while choosing each position from its own noise mixes them half
the time, as the pages' example says (page "Polymathic AI и исследователи из
Princeton выпустили FlashMap", section "Почему diffusion-драфтеры теряют в
доле принятых токенов?"; page "FlashMap并行草拟加速大模型解码", section
"一次猜 16 个 token，为什么还会前后不搭").  The semigroup check follows the
two-stage training described in section "一步生成整块，训练时做了什么" of the
same page: a flow map composes, X_{0.5,1} o X_{0,0.5} = X_{0,1}.
"""
import numpy as np

from oracle import flashmap as fm
from oracle import toy_flow as tf

K, V = 2, 4
T_END = 1.0 - 1e-6


def _tokens(x):
    """Per-position argmax of flattened blocks [n, K*V] (the oracle's token rule)."""
    blocks = x.reshape(-1, K, V)
    return np.array([[fm.argmax_lowest(b[i]) for i in range(K)] for b in blocks])


def _mixed(tok):
    good = {(0, 1), (2, 3)}
    return np.array([tuple(t) not in good for t in tok])


def test_shared_noise_never_mixes_factorised_mixes_half():
    n = 4000
    rng = np.random.default_rng(2024)
    x0 = rng.normal(size=(n, K * V))
    joint = _tokens(tf.flow(x0, 0.0, T_END))
    assert not _mixed(joint).any()
    # factorised: position i comes from the flow of its own independent noise
    xa = tf.flow(rng.normal(size=(n, K * V)), 0.0, T_END)
    xb = tf.flow(rng.normal(size=(n, K * V)), 0.0, T_END)
    fact = np.stack([_tokens(xa)[:, 0], _tokens(xb)[:, 1]], axis=1)
    frac = _mixed(fact).mean()
    assert abs(frac - 0.5) < 3 * np.sqrt(0.25 / n), frac


def test_semigroup_and_two_time_denoiser():
    rng = np.random.default_rng(7)
    x0 = rng.normal(size=(64, K * V))
    one = tf.flow(x0, 0.0, T_END)
    half = tf.flow(x0, 0.0, 0.5)
    two = tf.flow(half, 0.5, T_END)
    np.testing.assert_allclose(two, one, atol=1e-6)

    # The oracle's update is affine in D: X = x + alpha (D - x).  Read alpha
    # off the oracle and invert it to get the two-time denoiser D_{s,t} that
    # reproduces the exact map; as t -> s it must tend to the posterior mean
    # E[x1 | x_s], and at t = 1 it must be the endpoint itself.
    s = 0.5
    xs = half
    for t, tol in [(0.5 + 1e-4, 2e-3)]:
        e = np.ones_like(xs)
        alpha = (fm.flow_map_update(xs, xs + e, s, t) - xs)[0, 0]
        Xst = tf.flow(xs, s, t)
        D = xs + (Xst - xs) / alpha
        np.testing.assert_allclose(D, tf.posterior_mean(xs, s), atol=tol)
    np.testing.assert_allclose(fm.flow_map_update(xs, two, s, 1.0), two, atol=1e-15)

    # two oracle updates with the exact two-time denoisers land on X_{0,1}
    def denoiser(x, a, b):
        e = np.ones_like(x)
        al = (fm.flow_map_update(x, x + e, a, b) - x)[0, 0]
        return x + (tf.flow(x, a, b) - x) / al

    x = x0
    for a, b in [(0.0, 0.5), (0.5, T_END)]:
        x = fm.flow_map_update(x, denoiser(x, a, b), a, b)
    np.testing.assert_allclose(x, one, atol=1e-6)
    assert (_tokens(x) == _tokens(one)).all()
