"""The pins catch planted mistakes.

Each case copies the oracle's source, plants one plausible mistake (on the
CPU, in memory only), swaps the mutated function in and checks that at
least one pin fails.  This shows the pins are tight enough to trust the
oracle they pin.
"""
import inspect

import pytest

from oracle import flashmap as fm

import test_oracle_hand_draft as T1
import test_oracle_verify_exact as T4

SRC = inspect.getsource(fm)

VERIFY_MUTATIONS = {
    "ratio swapped": ("float(u_accept[j][i]) * q[y] < pp[y]", "float(u_accept[j][i]) * pp[y] < q[y]"),
    "no residual": ("r = np.maximum(pp - q, 0.0)", "r = pp.copy()"),
    "bonus from row K-1": ("_probs(target[alive[0], K], T)", "_probs(target[alive[0], K - 1], T)"),
    "alive set kept": ("alive = [j for j in alive if int(draft_tokens[j][i]) == accepted]", "pass"),
}

DRAFT_MUTATIONS = {
    "position sin/cos swapped": ("P[:, 0::2] = np.sin(i * w)", "P[:, 0::2] = np.cos(i * w)"),
    "no position term": ("x = z[j] + P", "x = z[j]"),
    "LM head transposed rows": ("out[j] = hf @ W[\"W_lm\"].T", "out[j] = (hf[:, ::-1] @ W[\"W_lm\"].T)"),
    "ties to highest": ("return int(np.argmax(row))", "return int(len(row) - 1 - np.argmax(row[::-1]))"),
}


def _mutated(name_a_b):
    a, b = name_a_b
    assert a in SRC
    ns = {}
    exec(compile(SRC.replace(a, b), "<mutant>", "exec"), ns)
    return ns


def _fails(fn):
    try:
        fn()
    except AssertionError:
        return True
    return False


@pytest.mark.parametrize("name", list(VERIFY_MUTATIONS))
def test_verify_mutation_is_caught(name, monkeypatch):
    ns = _mutated(VERIFY_MUTATIONS[name])
    monkeypatch.setattr(fm, "verify_sample", ns["verify_sample"])
    assert _fails(T4.test_lossless_tree_two_drafts_V4_K2)


@pytest.mark.parametrize("name", list(DRAFT_MUTATIONS))
def test_draft_mutation_is_caught(name, monkeypatch):
    ns = _mutated(DRAFT_MUTATIONS[name])
    for f in ("position_embedding", "dit_logits", "argmax_lowest", "draft"):
        monkeypatch.setattr(fm, f, ns[f])
    caught = _fails(T1.test_zero_dit_draft_matches_hand_values) or \
        _fails(T1.test_zero_dit_closed_form_any_noise)
    assert caught
