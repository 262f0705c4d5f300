"""Exact flow of a two-mode block distribution ("new york" / "san diego").

Test infrastructure only.  The pages motivate joint drafting with a
continuation that is either "new york" or "san diego" with equal chance: a
drafter that picks each position on its own mixes them ("new diego", "san
york") about half the time, while one noise sample mapped to a whole block
picks both positions together (P1 section "一次猜 16 个 token，为什么还会前后不搭";
P2 section "Почему diffusion-драфтеры теряют в доле принятых токенов?";
P4 section "Perché i drafter in diffusione perdono precisione?").

Here the data are K one-hot rows over a V-token vocabulary, flattened to
R^{K V}; noise x0 ~ N(0, I); the interpolant is x_t = (1-t) x0 + t x1.  For
a finite set of equally likely modes a_k the posterior mean is

    E[x1 | x_t = x] = sum_k w_k a_k,  w_k ∝ exp(-|x - t a_k|^2 / (2 (1-t)^2)),

and the flow ODE is dx/dt = (E[x1 | x] - x) / (1 - t).  The flow map
X_{s,t} is its solution operator, integrated here with adaptive RK45 in
fp64 over many samples at once.
"""
from __future__ import annotations

import numpy as np
from scipy.integrate import solve_ivp

VOCAB = ("new", "york", "san", "diego")
MODES = np.array([
    [[1, 0, 0, 0], [0, 1, 0, 0]],   # new york
    [[0, 0, 1, 0], [0, 0, 0, 1]],   # san diego
], dtype=np.float64)


def posterior_mean(x: np.ndarray, t: float, modes: np.ndarray = MODES) -> np.ndarray:
    """E[x1 | x_t = x] for x of shape [n, K*V]."""
    A = modes.reshape(len(modes), -1)
    d2 = ((x[:, None, :] - t * A[None, :, :]) ** 2).sum(-1)
    lw = -d2 / (2.0 * (1.0 - t) ** 2)
    lw -= lw.max(axis=1, keepdims=True)
    w = np.exp(lw)
    w /= w.sum(axis=1, keepdims=True)
    return w @ A


def flow(x: np.ndarray, s: float, t: float, modes: np.ndarray = MODES,
         rtol: float = 1e-10, atol: float = 1e-12) -> np.ndarray:
    """X_{s,t}(x) for x [n, K*V]; t may be at most 1 - 1e-6."""
    n, D = x.shape

    def rhs(tau, y):
        xx = y.reshape(n, D)
        return ((posterior_mean(xx, tau, modes) - xx) / (1.0 - tau)).ravel()

    sol = solve_ivp(rhs, (s, t), x.ravel(), method="RK45", rtol=rtol, atol=atol)
    if not sol.success:  # pragma: no cover
        raise RuntimeError(sol.message)
    return sol.y[:, -1].reshape(n, D)
