"""Seeded input generators: determinism, bf16 rounding, synthetic target statistic."""
import dataclasses

import numpy as np
import torch

import fm_synth as fs
from oracle import flashmap as fm


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).normal(size=100000).astype(np.float32) * 37.0
    x[:4] = [0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8]   # exact ties round to even
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(fs.bf16_bits(x), want)
    np.testing.assert_array_equal(fs.round_bf16(x), torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_generation_is_deterministic_and_chunked():
    a = fs.normal(77, (3, fs._CHUNK // 2 + 5), std=0.5)
    b = fs.normal(77, (3, fs._CHUNK // 2 + 5), std=0.5)
    np.testing.assert_array_equal(a, b)
    assert abs(a.std() - 0.5) < 1e-3
    c = fs.normal(78, (10,))
    assert not np.array_equal(c, fs.normal(77, (10,)))
    u = fs.uniform(5, (1000,))
    assert u.dtype == np.float64 and u.min() >= 0 and u.max() < 1


def test_weight_specs_param_count():
    # DiT blocks + adaLN + fc of the 8B-shaped drafter: about the 0.5B the
    # pages give for the Qwen3-8B drafter (E and LM head are frozen copies).
    s = fs.QWEN3_8B
    n = sum(int(np.prod(shp)) for name, shp in fs.weight_specs(s)
            if name not in ("E", "W_lm"))
    assert 0.45e9 < n < 0.55e9


def test_near_draft_target_accepted_length():
    # E[n] = sum_{i=1..16} a^i = 6.61 for a = 0.885; check the mean of 256
    # rounds against the exact distribution of n (geometric, capped at K).
    w = dataclasses.replace(fs.WORKLOADS["qwen3_8b_bs1"],
                            shape=dataclasses.replace(fs.QWEN3_8B, V=2048))
    K, a = w.shape.K, w.accept_a
    pk = np.array([a ** k * (1 - a) for k in range(K)] + [a ** K])
    mean = (np.arange(K + 1) * pk).sum()
    sd = np.sqrt(((np.arange(K + 1) - mean) ** 2 * pk).sum())
    assert abs(mean - 6.61) < 0.01
    rng = np.random.default_rng(1)
    ns = []
    for r in range(256):
        toks = rng.integers(0, w.shape.V, size=(1, 1, K))
        tgt = fs.target_logits(w, r, toks)
        n, _, _ = fm.verify_greedy(tgt[0], toks[0])
        ns.append(n)
    assert abs(np.mean(ns) - mean) < 3 * sd / np.sqrt(256)


def test_target_rows_shared_on_trie_prefix():
    w = dataclasses.replace(fs.WORKLOADS["qwen3_8b_2step_tree4"],
                            shape=dataclasses.replace(fs.QWEN3_8B, V=300))
    toks = np.zeros((1, 4, 16), dtype=np.int64)
    toks[0, 1, 3:] = 5          # shares the first 3 tokens with draft 0
    toks[0, 2, 0] = 7           # diverges at once
    toks[0, 3] = toks[0, 1]     # identical to draft 1
    t = fs.target_logits(w, 0, toks)
    for i in range(4):
        np.testing.assert_array_equal(t[0, 1, i], t[0, 0, i])
    assert not np.array_equal(t[0, 1, 4], t[0, 0, 4])
    np.testing.assert_array_equal(t[0, 2, 0], t[0, 0, 0])
    assert not np.array_equal(t[0, 2, 1], t[0, 0, 1])
    np.testing.assert_array_equal(t[0, 3], t[0, 1])
