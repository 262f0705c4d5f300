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
    "ties to highest": ("return int(ok[np.argmax(row[ok])])",
                        "return int(ok[len(ok) - 1 - np.argmax(row[ok][::-1])])"),
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


# ---- the two-step chain, the temperature and the argmax rule ----
import test_oracle_argmax as TA            # noqa: E402
import test_oracle_temperature as TT       # noqa: E402
import test_oracle_two_step as T6          # noqa: E402

CHAIN_MUTATIONS = {
    "intermediate softmax at the sampling temperature": (
        "x = flow_map_update(x, softmax(logits, 1.0), s, t)",
        "x = flow_map_update(x, softmax(logits, temperature if temperature > 0 else 1.0), s, t)"),
    "next step embeds D instead of the moved state": (
        "x = flow_map_update(x, softmax(logits, 1.0), s, t)", "x = softmax(logits, 1.0)"),
    "state not moved": ("x = flow_map_update(x, softmax(logits, 1.0), s, t)", "x = x"),
    "step size from swapped times": (
        "x = flow_map_update(x, softmax(logits, 1.0), s, t)",
        "x = flow_map_update(x, softmax(logits, 1.0), t, s)"),
    "every step conditioned on the first step's times": (
        "mods, final = conditioning(W, shape.n_blocks, s, t)",
        "mods, final = conditioning(W, shape.n_blocks, grid[0], grid[1])"),
    "start-time embedder fed the end time": (
        'te_s = W["W_ts2"] @ silu(W["W_ts1"] @ time_features(s))',
        'te_s = W["W_ts2"] @ silu(W["W_ts1"] @ time_features(t))'),
}

TEMPERATURE_MUTATIONS = {
    "draft sampling multiplies by T": (
        "return inverse_cdf(np.exp((z - z.max()) / T), u)",
        "return inverse_cdf(np.exp((z - z.max()) * T), u)"),
    "verify probabilities multiply by T": (
        "e = np.exp((z - z.max()) / T)\n    return e / e.sum()",
        "e = np.exp((z - z.max()) * T)\n    return e / e.sum()"),
}

ARGMAX_MUTATIONS = {
    "NaN may win": ("ok = np.flatnonzero(~np.isnan(row))", "ok = np.arange(row.size)"),
}


def _patch_all(ns, monkeypatch):
    for name, obj in ns.items():
        if callable(obj) and getattr(fm, name, None) is not None and not name.startswith("__"):
            monkeypatch.setattr(fm, name, obj)


@pytest.mark.parametrize("name", list(CHAIN_MUTATIONS))
def test_chain_mutation_is_caught(name, monkeypatch):
    _patch_all(_mutated(CHAIN_MUTATIONS[name]), monkeypatch)
    assert _fails(T6.test_two_step_sampled_matches_hand_values) or \
        _fails(T6.test_two_step_any_noise_matches_scalar_chain)


@pytest.mark.parametrize("name", list(TEMPERATURE_MUTATIONS))
def test_temperature_mutation_is_caught(name, monkeypatch):
    _patch_all(_mutated(TEMPERATURE_MUTATIONS[name]), monkeypatch)
    checks = [lambda: TT.test_two_token_sampling_threshold(2.0, 0.3),
              lambda: TT.test_point_mass_draft_accepts_below_tempered_probability(2.5),
              lambda: T4._check_lossless(V=4, K=2, N=2, seed=12, T=2.0)]
    assert any(_fails(c) for c in checks)


@pytest.mark.parametrize("name", list(ARGMAX_MUTATIONS))
def test_argmax_mutation_is_caught(name, monkeypatch):
    _patch_all(_mutated(ARGMAX_MUTATIONS[name]), monkeypatch)
    assert _fails(TA.test_nan_never_wins)


# ---- the prefix trie of the noise drafts ----
from oracle import tree as ot              # noqa: E402
import test_oracle_tree as TR              # noqa: E402

TREE_SRC = inspect.getsource(ot)
TREE_MUTATIONS = {
    "node key without its parent": (
        "key = (draft_node[j][i - 1] if i > 0 else -1, drafts[j][i])", "key = (-1, drafts[j][i])"),
    "a node is not its own ancestor": ("        u = v\n", "        u = parent[v]\n"),
    "node rows off by one": ("out[j, i] = node_rows[1 + draft_node[j][i - 1]]",
                             "out[j, i] = node_rows[draft_node[j][i - 1]]"),
}


@pytest.mark.parametrize("name", list(TREE_MUTATIONS))
def test_tree_mutation_is_caught(name, monkeypatch):
    a, b = TREE_MUTATIONS[name]
    assert a in TREE_SRC
    ns = {}
    exec(compile(TREE_SRC.replace(a, b), "<mutant>", "exec"), ns)
    for f in ("build_trie", "ancestors", "tree_attention", "draft_rows"):
        monkeypatch.setattr(ot, f, ns[f])
    checks = [TR.test_hand_built_trie, lambda: TR.test_trie_matches_brute_force_prefixes(3),
              TR.test_tree_attention_equals_causal_attention_on_each_path]
    assert any(_fails(c) for c in checks)
