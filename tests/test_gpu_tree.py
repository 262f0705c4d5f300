"""Target-side tree scoring on the GPU, against the oracle (exact for the
trie and the verify decisions, fp32 tolerance for the tree attention).

A tree of noise drafts is scored by the target once per unique prefix (page
"FlashMap并行草拟加速大模型解码", section "6.14 倍是最好成绩…").
"""
import os

import numpy as np
import pytest
import torch

import fm_synth as fs
from oracle import flashmap as om
from oracle import tree as ot
from step_flow_map_b200 import (FM_ERR_UNSUPPORTED, FlashmapError, fm_build_tree,
                                fm_tree_attention, fm_verify_greedy_tree, fm_verify_sample_tree)
from step_flow_map_b200.host import to_device

import gpu_util as gu

pytestmark = pytest.mark.gpu

GOLD = os.path.join(os.path.dirname(__file__), "golden", "t7_tree_of_four_drafts.txt")


def _drafts(seed, B, N, K, V):
    rng = np.random.default_rng(seed)
    d = rng.integers(0, V, size=(B, N, K))
    for b in range(B):
        for j in range(1, N):
            cut = int(rng.integers(0, K + 1))
            d[b, j, :cut] = d[b, int(rng.integers(0, j)), :cut]
    return d


def _gpu_tree(d):
    B, N, K = d.shape
    NN, W = N * K, (N * K + 63) // 64
    dev = "cuda"
    out = dict(token=torch.empty((B, NN), dtype=torch.int32, device=dev),
               parent=torch.empty((B, NN), dtype=torch.int32, device=dev),
               depth=torch.empty((B, NN), dtype=torch.int32, device=dev),
               n=torch.empty(B, dtype=torch.int32, device=dev),
               dn=torch.empty((B, N, K), dtype=torch.int32, device=dev),
               anc=torch.empty((B, NN, W), dtype=torch.int64, device=dev))
    fm_build_tree(to_device(d.astype(np.int32)), B, N, K, out["token"], out["parent"], out["depth"],
                  out["n"], out["dn"], out["anc"])
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("B,N,K,V,seed", [(3, 4, 16, 5, 1), (2, 7, 9, 3, 2), (1, 1, 16, 100, 3),
                                          (2, 32, 32, 2, 4)])
def test_build_tree_matches_oracle(B, N, K, V, seed):
    d = _drafts(seed, B, N, K, V)
    g = _gpu_tree(d)
    NN = N * K
    for b in range(B):
        token, parent, depth, dn = ot.build_trie(d[b])
        n = len(token)
        assert int(g["n"][b]) == n
        pad = [-1] * (NN - n)
        assert gu.to_np(g["token"][b]).tolist() == token + pad
        assert gu.to_np(g["parent"][b]).tolist() == parent + pad
        assert gu.to_np(g["depth"][b]).tolist() == depth + pad
        assert gu.to_np(g["dn"][b]).tolist() == dn
        anc = ot.ancestors(parent)
        words = gu.to_np(g["anc"][b]).view(np.uint64)
        for v in range(NN):
            got = {64 * k + bit for k in range(words.shape[1]) for bit in range(64)
                   if (int(words[v, k]) >> bit) & 1}
            assert got == (set(np.flatnonzero(anc[v]).tolist()) if v < n else set()), v


def test_build_tree_hand_example():
    rows = {}
    for line in open(GOLD):
        line = line.strip()
        if line and not line.startswith("#"):
            k, rest = line.split(None, 1)
            rows[k] = [[int(v) for v in r.split()] for r in rest.split(";")]
    d = np.array(rows["drafts"])[None]
    g = _gpu_tree(d)
    n = int(g["n"][0])
    assert gu.to_np(g["token"][0])[:n].tolist() == rows["token"][0]
    assert gu.to_np(g["parent"][0])[:n].tolist() == rows["parent"][0]
    assert gu.to_np(g["dn"][0]).tolist() == rows["draft_node"]


def test_tree_limits_are_checked_on_the_host():
    t = torch.zeros(8, dtype=torch.int32, device="cuda")
    for B, N, K in ((1, 33, 4), (1, 4, 300), (1, 1, 2**30)):
        with pytest.raises(FlashmapError) as e:
            fm_build_tree(t, B, N, K, t, t, t, t, t, t)
        assert e.value.status == FM_ERR_UNSUPPORTED


def test_tree_attention_matches_oracle():
    B, N, K, V, H, dh, L = 2, 4, 6, 3, 2, 40, 11
    d = _drafts(5, B, N, K, V)
    g = _gpu_tree(d)
    NN, D = N * K, H * dh
    rng = np.random.default_rng(6)
    q, kn, vn = (rng.normal(size=(B, NN, D)).astype(np.float32) for _ in range(3))
    kc, vc = (rng.normal(size=(B, L, D)).astype(np.float32) for _ in range(2))
    out = torch.zeros((B, NN, D), dtype=torch.float32, device="cuda")
    fm_tree_attention(to_device(q), to_device(kc), to_device(vc), to_device(kn), to_device(vn),
                      g["anc"], g["n"], B, NN, L, H, dh, out)
    got = gu.to_np(out)
    for b in range(B):
        _, parent, _, _ = ot.build_trie(d[b])
        n = len(parent)
        want = ot.tree_attention(q[b, :n].astype(np.float64), kc[b].astype(np.float64),
                                 vc[b].astype(np.float64), kn[b, :n].astype(np.float64),
                                 vn[b, :n].astype(np.float64), parent, H)
        np.testing.assert_allclose(got[b, :n], want, rtol=0, atol=1e-4)


def _node_targets(d, V, seed):
    # a synthetic target per trie node: N(0, 1.5^2), +20 on the next token of
    # the first draft through the node (the root: draft 0's first token)
    B, N, K = d.shape
    R = 1 + N * K
    rng = np.random.default_rng(seed)
    rows = (rng.normal(size=(B, R, V)) * 1.5).astype(np.float32)
    for b in range(B):
        _, _, _, dn = ot.build_trie(d[b])
        rows[b, 0, d[b, 0, 0]] += 20.0
        for j in range(N):
            for i in range(K - 1):
                if rng.random() < 0.9:
                    rows[b, 1 + dn[j][i], d[b, j, i + 1]] += 20.0 if j == 0 else 0.0
    return rows


def test_verify_tree_greedy_and_sampled_match_oracle():
    B, N, K, V = 3, 4, 16, 1000
    d = _drafts(8, B, N, K, 4)
    g = _gpu_tree(d)
    R = 1 + N * K
    rows = _node_targets(d, V, 9)
    w = fs.WORKLOADS["qwen3_8b_2step_tree4"]
    shape = fs.Shape(V=V, d=128, n_blocks=1, n_heads=1, mlp=128, K=K, hidden=8)
    import dataclasses
    ctx = gu.Context(shape, "f32", fs.make_weights(shape, "f32"), max_ctx=8, max_seqs=B,
                     max_noise=N, max_new=4)
    dv = to_device(d.astype(np.int32))
    n = torch.empty(B, dtype=torch.int32, device="cuda")
    br = torch.empty(B, dtype=torch.int32, device="cuda")
    out = torch.empty((B, K + 1), dtype=torch.int32, device="cuda")
    per_draft = np.stack([ot.draft_rows(rows[b], ot.build_trie(d[b])[3]) for b in range(B)])
    fm_verify_greedy_tree(ctx.ctx, to_device(rows), R, dv, g["dn"], B, N, K, V, n, br, out)
    want = gu.verify_oracle_all(per_draft, None, d, 0, None, None, True)
    np.testing.assert_array_equal(gu.to_np(n), want[0])
    np.testing.assert_array_equal(gu.to_np(br), want[1])
    np.testing.assert_array_equal(gu.to_np(out), want[2])
    assert want[0].max() > 0
    # stochastic, with a draft distribution per drafted position
    dlog = (np.random.default_rng(10).normal(size=(B, N, K, V)) * 1.0).astype(np.float32)
    ua = fs.uniform(93, (B, N, K))
    ur = fs.uniform(94, (B,))
    fm_verify_sample_tree(ctx.ctx, to_device(rows), R, to_device(dlog), dv, g["dn"], B, N, K, V, 0.9,
                          to_device(ua), to_device(ur), n, br, out)
    (wn, wb, wo), ties = gu.sample_tie_zone(per_draft, dlog, d, 0.9, ua, ur)
    ok = ~ties
    assert ok.sum() >= B - 1
    np.testing.assert_array_equal(gu.to_np(n)[ok], wn[ok])
    np.testing.assert_array_equal(gu.to_np(br)[ok], wb[ok])
    np.testing.assert_array_equal(gu.to_np(out)[ok], wo[ok])
    ctx.close()
