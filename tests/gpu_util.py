"""Helpers shared by the GPU parity tests (not collected by pytest)."""
from __future__ import annotations

import functools

import numpy as np
import torch

import fm_synth as fs
from oracle import flashmap as om
from step_flow_map_b200.host import Context, to_device

# Logit tolerances: |got - ref| <= ABS + REL * |ref|
TOL = {"bf16": (3e-2, 1e-2), "f32": (1e-4, 0.0)}
MARGIN = 0.1   # draft tokens must match where the oracle's top-1 - top-2 exceeds this


@functools.lru_cache(maxsize=2)
def weights(shape, dtype):
    return fs.make_weights(shape, dtype)


@functools.lru_cache(maxsize=1)
def weights64(shape, dtype):
    return {k: v.astype(np.float64) for k, v in weights(shape, dtype).items()}


def make_ctx(w: fs.Workload, max_new: int = 512, max_seqs: int | None = None) -> Context:
    return Context(w.shape, w.dtype, weights(w.shape, w.dtype), max_ctx=w.ctx + max(w.new_rows, 1) + 8,
                   max_seqs=max_seqs or w.B, max_noise=w.n_noise, max_new=max_new)


def gpu_prefill(ctx: Context, w: fs.Workload, seqs, max_new: int = 512):
    for b in seqs:
        h = fs.prefill_hidden(w, b)
        for p0 in range(0, w.ctx, max_new):
            part = to_device(h[p0:p0 + max_new][None], w.dtype)
            ctx.project([b], part, [p0])


def gpu_new_rows(ctx: Context, w: fs.Workload, r: int, seqs):
    if w.new_rows == 0:
        return
    ri = fs.round_inputs(w, r)
    ctx.project(list(seqs), to_device(ri.new_hidden[list(seqs)], w.dtype), [w.ctx] * len(seqs))


def oracle_kv(w: fs.Workload, b: int, r: int | None):
    W = weights64(w.shape, w.dtype)
    rows = fs.prefill_hidden(w, b)
    if r is not None and w.new_rows:
        rows = np.concatenate([rows, fs.round_inputs(w, r).new_hidden[b]], axis=0)
    _, kv = om.project_context(W, w.shape.n_blocks, rows)
    return kv


def oracle_draft(w: fs.Workload, b: int, r: int, kv=None):
    W = weights64(w.shape, w.dtype)
    kv = kv if kv is not None else oracle_kv(w, b, r)
    ri = fs.round_inputs(w, r)
    return om.draft(W, w.shape, kv, ri.noise[b], w.t_grid, w.temps[b], ri.u_draft[b])


def assert_logits_close(got: np.ndarray, want: np.ndarray, dtype: str, what=""):
    a, rel = TOL[dtype]
    err = np.abs(got.astype(np.float64) - want)
    bound = a + rel * np.abs(want)
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} logits out of tolerance; "
                           f"worst excess {(err - bound).max():.3g}, max err {err.max():.3g}")
    return float(err.max())


def assert_tokens_on_margin(got_tokens, want_logits, what=""):
    want_logits = np.asarray(want_logits)
    m = om.margins(want_logits)
    want = want_logits.argmax(-1)
    sure = m > MARGIN
    mism = (np.asarray(got_tokens) != want) & sure
    assert not mism.any(), f"{what}: {mism.sum()} draft tokens differ where margin > {MARGIN}"
    return int(sure.sum())


def sampled_token_sure(logits_row, T, u, frac=1e-6):
    """Oracle token of inverse-CDF sampling and whether u*total sits more than
    frac*total inside its CDF cell."""
    z = np.asarray(logits_row, dtype=np.float64)
    wts = np.exp((z - z.max()) / T)
    c = np.cumsum(wts)
    tot = c[-1]
    y = om.inverse_cdf(wts, u)
    lo = c[y - 1] if y > 0 else 0.0
    hi = c[y]
    t = u * tot
    return y, (t - lo) > frac * tot and (hi - t) > frac * tot


def sampled_token_near(logits_row, T, u, token, tol=2e-4):
    """True when the oracle's CDF cell of `token` lies within tol*total of u*total:
    a draw from logits that differ from the oracle's by the bf16 tolerance."""
    z = np.asarray(logits_row, dtype=np.float64)
    wts = np.exp((z - z.max()) / T)
    c = np.cumsum(wts)
    tot = c[-1]
    lo = c[token - 1] if token > 0 else 0.0
    hi = c[token]
    t = u * tot
    return lo - tol * tot <= t <= hi + tol * tot


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def verify_oracle_all(target, dlog, draft, T, ua, ures, greedy: bool):
    """Oracle verify of every sequence; returns (n, branch, out [B, K+1] -1 padded)."""
    B, N, K1, V = target.shape
    n = np.zeros(B, np.int64)
    br = np.zeros(B, np.int64)
    out = -np.ones((B, K1), np.int64)
    for b in range(B):
        if greedy:
            nb, bb, toks = om.verify_greedy(target[b], draft[b])
        else:
            nb, bb, toks = om.verify_sample(target[b], None if dlog is None else dlog[b], draft[b],
                                            T, ua[b], ures[b])
        n[b], br[b] = nb, bb
        out[b, :len(toks)] = toks
    return n, br, out


def sample_tie_zone(target, dlog, draft, T, ua, ures, eps=1e-9):
    """Sequences whose oracle decision changes when every uniform moves by eps."""
    B = target.shape[0]
    base = verify_oracle_all(target, dlog, draft, T, ua, ures, False)
    ties = np.zeros(B, bool)
    for sgn in (-1, 1):
        alt = verify_oracle_all(target, dlog, draft, T, np.clip(ua + sgn * eps, 0, 1 - 1e-16),
                                np.clip(ures + sgn * eps, 0, 1 - 1e-16), False)
        for k in range(3):
            ties |= np.atleast_2d((alt[k] != base[k]).reshape(B, -1)).any(axis=1)
    return base, ties
