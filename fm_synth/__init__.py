"""Seeded synthetic inputs shared by the fp64 oracle and the CUDA path.

This module only draws random numbers and rounds them to bf16.  It computes
no step of the drafter or of the verifier, so the oracle and the GPU path can
both take their inputs from it without sharing any of the method's
arithmetic.

Workloads (shapes follow the pages: K = 16 block slots, a 6-block DiT with
embedding width 2048 and 16 heads, vocabulary 151,936, five tapped target
layers -- page "FlashMap并行草拟加速大模型解码", section
"一步生成整块，训练时做了什么"; page "Polymathic AI и исследователи из
Princeton выпустили FlashMap", section "Как работает FlashMap?"):

* ``tiny_f32``      V=512, d=128, 2 blocks, 4 heads, MLP 512, hidden 256, ctx 32
* ``qwen3_4b_bs1``  V=151936, d=2048, 6 blocks, 16 heads, MLP 8192, hidden 2560, ctx 512
* ``qwen3_8b_bs1``  as above with hidden 4096, ctx 1024 (the concurrency-1 bench)
* ``qwen3_8b_2step_tree4``  two steps (0, 0.5, 1), 4 noise drafts, T=1, ctx 2048
* ``qwen3_8b_bs64`` 64 sequences, ctx 4096, 32 greedy + 32 sampled at T=1
* ``qwen3_8b_bs64_ctx256`` the same with 256 context rows (profiler captures)

Seeds: weights use ``1000 + tensor_index``; round ``r`` draws its noise from
``2000 + r``, its new context rows from ``3000 + r``, its target-logit
perturbation from ``4000 + r`` and its uniforms from ``5000 + r``.  The
prefill context of sequence b uses seed 2999, stream b.  Every draw is PCG64 through a
``SeedSequence``, split into fixed chunks so that large tensors can be drawn
on several threads with identical results.
"""
from __future__ import annotations

import concurrent.futures as _cf
import os
from dataclasses import dataclass, field

import numpy as np

WEIGHT_STD = 0.02
TIME_FREQ_DIM = 256
_CHUNK = 1 << 24  # elements per independently seeded chunk


# --------------------------------------------------------------------------
# bf16 rounding (round to nearest even), done on the fp32 bit pattern.
# --------------------------------------------------------------------------
def bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 array -> uint16 bf16 bit patterns, round-to-nearest-even."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns -> fp32 values (exact)."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_bf16(a: np.ndarray) -> np.ndarray:
    """fp32 values rounded to the nearest bf16, returned as fp32."""
    return bf16_to_f32(bf16_bits(a))


# --------------------------------------------------------------------------
# Shapes and workloads
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class Shape:
    V: int
    d: int
    n_blocks: int
    n_heads: int
    mlp: int
    K: int
    hidden: int
    n_taps: int = 5

    @property
    def dh(self) -> int:
        return self.d // self.n_heads


@dataclass(frozen=True)
class Workload:
    name: str
    shape: Shape
    dtype: str            # "f32" or "bf16": storage type of weights/noise/hidden
    B: int                # sequences
    n_noise: int          # noise drafts per sequence
    ctx: int              # prefill context rows per sequence
    new_rows: int         # context rows appended per round
    t_grid: tuple         # model-time grid, 0 -> 1
    temps: tuple          # per-sequence temperature (0 = greedy)
    target: str           # "gaussian" or "near_draft"
    target_std: float
    accept_a: float = 0.885   # chance the boosted target token is the drafted one
    boost: float = 20.0
    rounds: int = 1
    description: str = ""

    @property
    def M(self) -> int:
        return self.B * self.n_noise * self.shape.K


TINY = Shape(V=512, d=128, n_blocks=2, n_heads=4, mlp=512, K=16, hidden=256)
QWEN3_4B = Shape(V=151936, d=2048, n_blocks=6, n_heads=16, mlp=8192, K=16, hidden=2560)
QWEN3_8B = Shape(V=151936, d=2048, n_blocks=6, n_heads=16, mlp=8192, K=16, hidden=4096)

WORKLOADS = {
    "tiny_f32": Workload(
        "tiny_f32", TINY, "f32", B=1, n_noise=1, ctx=32, new_rows=0,
        t_grid=(0.0, 1.0), temps=(0.0,), target="gaussian", target_std=2.0,
        rounds=4, description="tiny fp32 drafter, greedy verify vs N(0,2^2) target"),
    "qwen3_4b_bs1": Workload(
        "qwen3_4b_bs1", QWEN3_4B, "bf16", B=1, n_noise=1, ctx=512, new_rows=17,
        t_grid=(0.0, 1.0), temps=(0.0,), target="near_draft", target_std=1.5,
        rounds=4, description="Qwen3-4B-shaped drafter, bf16, batch 1, greedy"),
    "qwen3_8b_bs1": Workload(
        "qwen3_8b_bs1", QWEN3_8B, "bf16", B=1, n_noise=1, ctx=1024, new_rows=17,
        t_grid=(0.0, 1.0), temps=(0.0,), target="near_draft", target_std=1.5,
        rounds=256, description="Qwen3-8B-shaped drafter, bf16, batch 1, greedy, 256 rounds"),
    "qwen3_8b_2step_tree4": Workload(
        "qwen3_8b_2step_tree4", QWEN3_8B, "bf16", B=1, n_noise=4, ctx=2048, new_rows=17,
        t_grid=(0.0, 0.5, 1.0), temps=(1.0,), target="near_draft", target_std=1.5,
        rounds=4, description="two steps, 4 noise drafts as a tree, T=1 sampling"),
    "qwen3_8b_bs64": Workload(
        "qwen3_8b_bs64", QWEN3_8B, "bf16", B=64, n_noise=1, ctx=4096, new_rows=17,
        t_grid=(0.0, 1.0), temps=tuple([0.0] * 32 + [1.0] * 32), target="near_draft",
        target_std=1.5, rounds=1, description="64 sequences x K=16, mixed greedy / T=1"),
    # the same M = 1024 GEMMs with 256 context rows: small enough on the
    # device for a full-metric profiler capture
    "qwen3_8b_bs64_ctx256": Workload(
        "qwen3_8b_bs64_ctx256", QWEN3_8B, "bf16", B=64, n_noise=1, ctx=256, new_rows=17,
        t_grid=(0.0, 1.0), temps=tuple([0.0] * 32 + [1.0] * 32), target="near_draft",
        target_std=1.5, rounds=1, description="as qwen3_8b_bs64 with 256 context rows"),
}


# --------------------------------------------------------------------------
# Random streams
# --------------------------------------------------------------------------
def _gen(seed, *sub) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), *map(int, sub)])))


def _threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def normal(seed, shape, std=1.0, sub=0) -> np.ndarray:
    """fp32 N(0, std^2) array drawn in fixed chunks, each with its own stream."""
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) if shape else 1
    out = np.empty(n, dtype=np.float32)
    chunks = [(i, min(n, i + _CHUNK)) for i in range(0, n, _CHUNK)]

    def fill(ci):
        a, b = chunks[ci]
        _gen(seed, sub, ci).standard_normal(b - a, dtype=np.float32, out=out[a:b])
        if std != 1.0:
            out[a:b] *= np.float32(std)

    if len(chunks) > 1:
        with _cf.ThreadPoolExecutor(min(_threads(), len(chunks))) as ex:
            list(ex.map(fill, range(len(chunks))))
    elif chunks:
        fill(0)
    return out.reshape(shape)


def uniform(seed, shape, sub=0) -> np.ndarray:
    """fp64 uniforms in [0, 1)."""
    return _gen(seed, sub).random(tuple(int(s) for s in shape), dtype=np.float64)


def _store(a: np.ndarray, dtype: str) -> np.ndarray:
    return round_bf16(a) if dtype == "bf16" else a.astype(np.float32, copy=False)


# --------------------------------------------------------------------------
# Weights
# --------------------------------------------------------------------------
def weight_specs(s: Shape):
    """(name, shape) in tensor-index order.  Linear weights are [out, in]."""
    d = s.d
    specs = [
        ("E", (s.V, d)),                       # soft-embedding table, row per token
        ("W_lm", (s.V, d)),                    # LM head, row per token
        ("W_fc", (d, s.n_taps * s.hidden)),    # context projection
        ("W_ts1", (d, TIME_FREQ_DIM)), ("W_ts2", (d, d)),   # embedder of time s
        ("W_tt1", (d, TIME_FREQ_DIM)), ("W_tt2", (d, d)),   # embedder of time t
        ("W_ada_f", (2 * d, d)),               # final shift / scale
    ]
    for l in range(s.n_blocks):
        specs += [
            (f"W_qkv.{l}", (3 * d, d)),
            (f"W_o.{l}", (d, d)),
            (f"W_up.{l}", (s.mlp, d)),
            (f"W_down.{l}", (d, s.mlp)),
            (f"W_ada.{l}", (6 * d, d)),
        ]
    return specs


def make_weights(s: Shape, dtype: str, std: float = WEIGHT_STD) -> dict:
    """All weights as fp32 arrays holding exactly the stored values."""
    return {name: _store(normal(1000 + i, shp, std), dtype)
            for i, (name, shp) in enumerate(weight_specs(s))}


# --------------------------------------------------------------------------
# Per-round inputs
# --------------------------------------------------------------------------
@dataclass
class RoundInputs:
    noise: np.ndarray        # [B, N, K, V]   fp32 values (bf16-exact when bf16)
    new_hidden: np.ndarray   # [B, new_rows, n_taps, hidden]
    u_draft: np.ndarray      # [B, N, K] fp64, draft sampling
    u_accept: np.ndarray     # [B, N, K] fp64, verify accept tests
    u_res: np.ndarray        # [B] fp64, residual / bonus draw
    extra: dict = field(default_factory=dict)


def prefill_hidden(w: Workload, b: int) -> np.ndarray:
    """Prefill context of sequence b: [ctx, n_taps, hidden] target hidden states, N(0,1)."""
    s = w.shape
    return _store(normal(2999, (w.ctx, s.n_taps, s.hidden), sub=b), w.dtype)


def round_inputs(w: Workload, r: int) -> RoundInputs:
    s = w.shape
    noise = _store(normal(2000 + r, (w.B, w.n_noise, s.K, s.V)), w.dtype)
    hid = _store(normal(3000 + r, (w.B, w.new_rows, s.n_taps, s.hidden)), w.dtype)
    u_draft = uniform(5000 + r, (w.B, w.n_noise, s.K), sub=0)
    u_accept = uniform(5000 + r, (w.B, w.n_noise, s.K), sub=1)
    u_res = uniform(5000 + r, (w.B,), sub=2)
    return RoundInputs(noise, hid, u_draft, u_accept, u_res)


def factorised_noise(w: Workload, r: int) -> np.ndarray:
    """[B, K, K, V] noise of round r for factorised drafting: block i drafts
    position i only, each block an independent N(0, 1) draw (seed 2000 + r,
    stream 1; the joint draft of the same round uses stream 0)."""
    s = w.shape
    return _store(normal(2000 + r, (w.B, s.K, s.K, s.V), sub=1), w.dtype)


def target_logits(w: Workload, r: int, draft_tokens: np.ndarray,
                  draft_logits: np.ndarray | None = None) -> np.ndarray:
    """Synthetic target rows [B, N, K+1, V] fp32 standing in for the target model.

    ``gaussian``: N(0, target_std^2) everywhere, independent of the draft.

    ``near_draft``: row i of draft j is ``base + N(0, target_std^2)`` plus
    ``boost`` on one chosen token.  ``base`` is the draft's own logit row
    (zero for the bonus row K).  The chosen token is the drafted token with
    chance ``accept_a`` and otherwise a uniformly drawn different token, so
    the expected greedy accepted length is sum_{i=1..K} a^i.  Rows are made
    per prefix-trie node: a draft whose first i tokens equal those of an
    earlier draft copies that draft's row i, so drafts that share a prefix
    see the same target distribution there.
    """
    s = w.shape
    B, N, K, V = w.B, w.n_noise, s.K, s.V
    noise = normal(4000 + r, (B, N, K + 1, V), std=w.target_std)
    if w.target == "gaussian":
        return noise
    g = _gen(4000 + r, 7)
    coins = g.random((B, N, K + 1))
    alt = g.integers(0, V - 1, size=(B, N, K + 1))
    out = noise
    tok = np.asarray(draft_tokens).reshape(B, N, K)
    for b in range(B):
        for j in range(N):
            for i in range(K + 1):
                row = out[b, j, i]
                if i < K:
                    if draft_logits is not None:
                        row += np.asarray(draft_logits[b, j, i], dtype=np.float32)
                    y = int(tok[b, j, i])
                    c = y if coins[b, j, i] < w.accept_a else int(alt[b, j, i]) + (int(alt[b, j, i]) >= y)
                else:
                    c = int(alt[b, j, i])
                row[c] += np.float32(w.boost)
    # per-trie-node sharing: row i depends on the prefix tokens [0, i)
    for b in range(B):
        for j in range(1, N):
            for i in range(K + 1):
                for j0 in range(j):
                    if np.array_equal(tok[b, j0, :i], tok[b, j, :i]):
                        out[b, j, i] = out[b, j0, i]
                        break
    return out
