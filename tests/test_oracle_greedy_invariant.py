"""Greedy speculative decoding reproduces plain greedy target decoding.

The pages state that with a correct verifier greedy output is the same as
ordinary target-model decoding (page "FlashMap Drafts 16 Dependent Tokens at
Once…", section "Why drafting still costs time"; page "Polymathic AI и
исследователи из Princeton выпустили FlashMap", section "Что такое
FlashMap?").  The toy target is a deterministic next-token table; drafts are
random, adversarial (always wrong) and perfect.
"""
import numpy as np
import pytest

from oracle import flashmap as fm

V, K, STEPS = 97, 16, 200


def _table(seed):
    return np.random.default_rng(seed).normal(size=(V, V))


def _plain(table, start, n):
    out, last = [], start
    for _ in range(n):
        last = int(np.argmax(table[last]))
        out.append(last)
    return out


def _spec(table, start, n, drafter):
    out, last, rounds = [], start, 0
    while len(out) < n:
        y = drafter(last, out)
        prefix = [last] + list(y)
        target = np.array([table[prefix[i]] for i in range(K + 1)])[None]
        acc, _, toks = fm.verify_greedy(target, [y])
        assert len(toks) == acc + 1
        out.extend(toks)
        last = toks[-1]
        rounds += 1
    return out[:n], rounds


@pytest.mark.parametrize("kind", ["random", "adversarial", "perfect", "half"])
def test_spec_equals_plain_greedy(kind):
    table = _table(7)
    rng = np.random.default_rng(8)
    plain = _plain(table, 3, STEPS)

    def drafter(last, out):
        truth = _plain(table, last, K)
        if kind == "random":
            return [int(v) for v in rng.integers(0, V, size=K)]
        if kind == "adversarial":
            return [(t + 1) % V for t in truth]
        if kind == "perfect":
            return truth
        cut = int(rng.integers(0, K + 1))
        return truth[:cut] + [(t + 1) % V for t in truth[cut:]]

    spec, rounds = _spec(table, 3, STEPS, drafter)
    assert spec == plain
    if kind == "perfect":
        assert rounds == -(-STEPS // (K + 1))
    if kind == "adversarial":
        assert rounds == STEPS
