"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Tolerances: draft logits |d| <= 3e-2 + 1e-2 |ref| (bf16 storage) or 1e-4
(fp32); greedy draft tokens equal wherever the oracle's top-1/top-2 margin
exceeds 0.1; sampled draft tokens equal (fp32) wherever u sits more than
1e-6 of the mass inside its CDF cell, or (bf16) lie within 2e-4 of the mass
of u's place in the oracle's CDF; verify outputs (accepted length, branch,
tokens) bit-exact on the same logits and uniforms, except decisions within
1e-9 of a threshold, which are reported and skipped.
"""
import dataclasses

import numpy as np
import pytest
import torch

import fm_synth as fs
from oracle import flashmap as om
import step_flow_map_b200 as fmb
from step_flow_map_b200 import FM_ERR_ARG, FlashmapError
from step_flow_map_b200.host import to_device

import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    torch.cuda.synchronize()


# ------------------------------------------------------------------ tiny fp32, end to end
def test_tiny_f32_rounds():
    w = gu.fs.WORKLOADS["tiny_f32"]
    ctx = gu.make_ctx(w)
    gu.gpu_prefill(ctx, w, [0])
    kv = gu.oracle_kv(w, 0, None)
    for r in range(w.rounds):
        ri = fs.round_inputs(w, r)
        tok, lg = ctx.draft([0], to_device(ri.noise, "f32"), w.t_grid, w.temps)
        ref = gu.oracle_draft(w, 0, r, kv)
        gu.assert_logits_close(gu.to_np(lg)[0], ref["logits"], "f32", f"round {r}")
        gu.assert_tokens_on_margin(gu.to_np(tok)[0], ref["logits"], f"round {r}")
        # greedy verify on the oracle's own draft
        tgt = fs.target_logits(w, r, ref["tokens"][None])
        n, br, out = ctx.verify_greedy(to_device(tgt, "f32"),
                                       to_device(ref["tokens"][None].astype(np.int32)))
        want = gu.verify_oracle_all(tgt, None, ref["tokens"][None], 0, None, None, True)
        np.testing.assert_array_equal(gu.to_np(n), want[0])
        np.testing.assert_array_equal(gu.to_np(br), want[1])
        np.testing.assert_array_equal(gu.to_np(out), want[2])
    ctx.close()


@pytest.mark.parametrize("T,N,grid", [(1.0, 2, (0.0, 1.0)), (0.7, 1, (0.0, 0.5, 1.0))])
def test_tiny_f32_sampled_draft_exact(T, N, grid):
    # fp32 logits agree with the oracle to ~1e-6, far below a CDF cell of a
    # 512-token softmax, so the inverse-CDF draw must match exactly
    w = dataclasses.replace(gu.fs.WORKLOADS["tiny_f32"], n_noise=N, t_grid=grid, temps=(T,))
    ctx = gu.make_ctx(w)
    gu.gpu_prefill(ctx, w, [0])
    kv = gu.oracle_kv(w, 0, None)
    checked = 0
    for r in range(3):
        ri = fs.round_inputs(w, r)
        tok, lg = ctx.draft([0], to_device(ri.noise, "f32"), w.t_grid, w.temps,
                            u_draft=to_device(ri.u_draft))
        ref = gu.oracle_draft(w, 0, r, kv)
        gu.assert_logits_close(gu.to_np(lg)[0], ref["logits"], "f32", f"round {r}")
        got = gu.to_np(tok)[0]
        for j in range(N):
            for i in range(w.shape.K):
                y, sure = gu.sampled_token_sure(ref["logits"][j, i], T, ri.u_draft[0, j, i])
                assert y == ref["tokens"][j, i]
                if sure:
                    checked += 1
                    assert got[j, i] == y, (r, j, i)
    assert checked >= 40
    ctx.close()


# ------------------------------------------------------------------ verify kernels
def _verify_case(V, B, N, K, seed, share=True):
    w = dataclasses.replace(fs.WORKLOADS["qwen3_8b_2step_tree4"], B=B, n_noise=N,
                            shape=dataclasses.replace(fs.QWEN3_8B, V=V, K=K))
    rng = np.random.default_rng(seed)
    tok = rng.integers(0, V, size=(B, N, K))
    if share and N > 1:
        for b in range(B):
            for j in range(1, N):
                cut = int(rng.integers(0, K + 1))
                tok[b, j, :cut] = tok[b, 0, :cut]
    dlog = fs.normal(777 + seed, (B, N, K, V))
    tgt = fs.target_logits(w, seed, tok, dlog)
    return w, tok, dlog, tgt


@pytest.mark.parametrize("B,N", [(5, 1), (3, 4), (1, 1)])
def test_verify_greedy_exact(B, N):
    V, K = 151936, 16
    w, tok, _, tgt = _verify_case(V, B, N, K, seed=10 + B + N)
    ctx = gu.make_ctx(dataclasses.replace(w, ctx=4, new_rows=1), max_new=4)
    n, br, out = ctx.verify_greedy(to_device(tgt), to_device(tok.astype(np.int32)))
    want = gu.verify_oracle_all(tgt, None, tok, 0, None, None, True)
    np.testing.assert_array_equal(gu.to_np(n), want[0])
    np.testing.assert_array_equal(gu.to_np(br), want[1])
    np.testing.assert_array_equal(gu.to_np(out), want[2])
    assert want[0].max() > 0
    ctx.close()


def test_verify_greedy_nan_rows():
    # NaN never wins (it ranks below -inf); a row of NaN gives token 0
    V, K, B = 2053, 16, 3
    w = dataclasses.replace(fs.WORKLOADS["qwen3_8b_bs1"], B=B,
                            shape=dataclasses.replace(fs.QWEN3_8B, V=V, K=K))
    rng = np.random.default_rng(9)
    tgt = rng.normal(size=(B, 1, K + 1, V)).astype(np.float32)
    tok = tgt.argmax(-1)[:, :, :K].astype(np.int64)
    tgt[0, 0, 2, tok[0, 0, 2]] = np.nan          # the argmax itself turns NaN: n = 2
    tgt[1, 0, 0, :] = np.nan
    tok[1, 0, 0] = 0
    tgt[2, 0, 4, :] = -np.inf
    tgt[2, 0, 4, :100] = np.nan
    tok[2, 0, 4] = 100
    ctx = gu.make_ctx(dataclasses.replace(w, ctx=4, new_rows=1), max_new=4)
    n, br, out = ctx.verify_greedy(to_device(tgt), to_device(tok.astype(np.int32)))
    want = gu.verify_oracle_all(tgt, None, tok, 0, None, None, True)
    np.testing.assert_array_equal(gu.to_np(n), want[0])
    np.testing.assert_array_equal(gu.to_np(out), want[2])
    assert list(want[0]) == [2, 16, 16]
    ctx.close()


def test_verify_greedy_ties_and_ragged_vocab():
    # constant rows: every index ties, the lowest wins; odd V leaves a ragged tail
    V, K, B = 1001, 16, 2
    w = dataclasses.replace(fs.WORKLOADS["qwen3_8b_bs1"], B=B,
                            shape=dataclasses.replace(fs.QWEN3_8B, V=V, K=K))
    tgt = np.zeros((B, 1, K + 1, V), np.float32)
    tgt[1, 0, :, V - 1] = 1.0              # argmax at the very last entry
    tok = np.zeros((B, 1, K), np.int64)
    tok[1] = V - 1
    tok[0, 0, 5] = 3
    ctx = gu.make_ctx(dataclasses.replace(w, ctx=4, new_rows=1), max_new=4)
    n, br, out = ctx.verify_greedy(to_device(tgt), to_device(tok.astype(np.int32)))
    want = gu.verify_oracle_all(tgt, None, tok, 0, None, None, True)
    np.testing.assert_array_equal(gu.to_np(n), want[0])
    np.testing.assert_array_equal(gu.to_np(out), want[2])
    assert list(want[0]) == [5, 16]
    ctx.close()


@pytest.mark.parametrize("B,N,T,with_q", [(4, 1, 1.0, True), (3, 4, 1.0, True),
                                          (2, 4, 0.7, True), (3, 1, 1.0, False)])
def test_verify_sample_exact(B, N, T, with_q):
    V, K = 151936, 16
    w, tok, dlog, tgt = _verify_case(V, B, N, K, seed=20 + B + N)
    ua = fs.uniform(91, (B, N, K))
    ur = fs.uniform(92, (B,))
    dl = dlog if with_q else None
    ctx = gu.make_ctx(dataclasses.replace(w, ctx=4, new_rows=1), max_new=4)
    n, br, out = ctx.verify_sample(to_device(tgt), None if dl is None else to_device(dl),
                                   to_device(tok.astype(np.int32)), T, to_device(ua), to_device(ur))
    (wn, wb, wo), ties = gu.sample_tie_zone(tgt, dl, tok, T, ua, ur)
    ok = ~ties
    assert ok.sum() >= B - 1
    np.testing.assert_array_equal(gu.to_np(n)[ok], wn[ok])
    np.testing.assert_array_equal(gu.to_np(br)[ok], wb[ok])
    np.testing.assert_array_equal(gu.to_np(out)[ok], wo[ok])
    ctx.close()


# ------------------------------------------------------------------ bf16 drafts at full size
@pytest.mark.parametrize("name", ["qwen3_8b_bs1", "qwen3_4b_bs1"])
def test_bf16_draft_full_size(name):
    w = fs.WORKLOADS[name]
    ctx = gu.make_ctx(w)
    gu.gpu_prefill(ctx, w, [0])
    r = 0
    gu.gpu_new_rows(ctx, w, r, [0])
    ri = fs.round_inputs(w, r)
    tok, lg = ctx.draft([0], to_device(ri.noise, "bf16"), w.t_grid, w.temps)
    ref = gu.oracle_draft(w, 0, r)
    gu.assert_logits_close(gu.to_np(lg)[0], ref["logits"], "bf16", name)
    sure = gu.assert_tokens_on_margin(gu.to_np(tok)[0], ref["logits"], name)
    assert sure >= 4
    # greedy verify on oracle-made inputs
    tgt = fs.target_logits(w, r, ref["tokens"][None], ref["logits"][None].astype(np.float32))
    n, br, out = ctx.verify_greedy(to_device(tgt), to_device(ref["tokens"][None].astype(np.int32)))
    want = gu.verify_oracle_all(tgt, None, ref["tokens"][None], 0, None, None, True)
    np.testing.assert_array_equal(gu.to_np(n), want[0])
    np.testing.assert_array_equal(gu.to_np(out), want[2])
    ctx.close()


def test_two_step_tree_sampled():
    w = fs.WORKLOADS["qwen3_8b_2step_tree4"]
    ctx = gu.make_ctx(w)
    gu.gpu_prefill(ctx, w, [0])
    r = 0
    gu.gpu_new_rows(ctx, w, r, [0])
    ri = fs.round_inputs(w, r)
    tok, lg = ctx.draft([0], to_device(ri.noise, "bf16"), w.t_grid, w.temps,
                        u_draft=to_device(ri.u_draft))
    ref = gu.oracle_draft(w, 0, r)
    gu.assert_logits_close(gu.to_np(lg)[0], ref["logits"], "bf16", "two-step final logits")
    got = gu.to_np(tok)[0]
    # bf16 logits move CDF cells of a 151,936-token softmax by about one cell
    # width, so sampled tokens are checked for lying at u's place in the
    # oracle's CDF up to that tolerance (exact sampling is pinned on fp32)
    for j in range(w.n_noise):
        for i in range(w.shape.K):
            assert gu.sampled_token_near(ref["logits"][j, i], 1.0, ri.u_draft[0, j, i],
                                         int(got[j, i])), (j, i)
    # tree stochastic verify on oracle-made inputs
    dl = ref["logits"][None].astype(np.float32)
    tgt = fs.target_logits(w, r, ref["tokens"][None], dl)
    n, br, out = ctx.verify_sample(to_device(tgt), to_device(dl),
                                   to_device(ref["tokens"][None].astype(np.int32)), 1.0,
                                   to_device(ri.u_accept), to_device(ri.u_res))
    (wn, wb, wo), ties = gu.sample_tie_zone(tgt, dl, ref["tokens"][None], 1.0, ri.u_accept, ri.u_res)
    if not ties[0]:
        assert (int(gu.to_np(n)[0]), int(gu.to_np(br)[0])) == (wn[0], wb[0])
        np.testing.assert_array_equal(gu.to_np(out)[0], wo[0])
    ctx.close()


def test_bench_path_8b_bs1_fused_argmax_rounds():
    # the exact path the concurrency-1 bench times: the round's new context
    # rows projected inside the persistent DiT pass, then the LM head with
    # the fused per-tile argmax (no logits written) and the token selection
    # over its 1,187 tile partials -- over four rounds whose appended rows
    # accumulate in the cache
    w = fs.WORKLOADS["qwen3_8b_bs1"]
    rounds = 4
    ctx = gu.Context(w.shape, w.dtype, gu.weights(w.shape, w.dtype),
                     max_ctx=w.ctx + rounds * w.new_rows + 8, max_seqs=1, max_noise=1, max_new=512)
    gu.gpu_prefill(ctx, w, [0])
    rows = [fs.prefill_hidden(w, 0)]
    W = gu.weights64(w.shape, w.dtype)
    checked = 0
    for r in range(rounds):
        ri = fs.round_inputs(w, r)
        ctx.project([0], to_device(ri.new_hidden, "bf16"), [w.ctx + r * w.new_rows])
        rows.append(ri.new_hidden[0])
        tok, none = ctx.draft([0], to_device(ri.noise, "bf16"), w.t_grid, w.temps, logits=False)
        assert none is None
        _, kv = om.project_context(W, w.shape.n_blocks, np.concatenate(rows, axis=0))
        ref = om.draft(W, w.shape, kv, ri.noise[0], w.t_grid)
        checked += gu.assert_tokens_on_margin(gu.to_np(tok)[0], ref["logits"], f"round {r}")
        # no bounded wait inside the pass gave up (an aborted pass leaves
        # stale tokens that can still fall outside the checked margin)
        fmb.fm_device_status(ctx.ctx)
    assert checked >= 8
    ctx.close()


# sequences of the batch-64 round checked against the oracle: both halves
# (greedy 0..31, sampled 32..63) and every 128-row activation tile; the
# oracle projects 4,113 context rows per sequence, so the whole batch would
# take minutes on the host
BS64_CHECK = (0, 5, 13, 21, 30, 31, 32, 33, 40, 47, 55, 63)


def test_bs64_mixed_sampled_rows():
    w = fs.WORKLOADS["qwen3_8b_bs64"]
    ctx = gu.make_ctx(w, max_new=1024)
    seqs = list(range(w.B))
    gu.gpu_prefill(ctx, w, seqs, max_new=1024)
    r = 0
    gu.gpu_new_rows(ctx, w, r, seqs)
    ri = fs.round_inputs(w, r)
    tok, lg = ctx.draft(seqs, to_device(ri.noise, "bf16"), w.t_grid, w.temps,
                        u_draft=to_device(ri.u_draft))
    lg_np = gu.to_np(lg)
    tok_np = gu.to_np(tok)
    for b in BS64_CHECK:
        ref = gu.oracle_draft(w, b, r)
        gu.assert_logits_close(lg_np[b], ref["logits"], "bf16", f"bs64 seq {b}")
        if w.temps[b] == 0:
            gu.assert_tokens_on_margin(tok_np[b], ref["logits"], f"bs64 seq {b}")
        else:
            for i in range(w.shape.K):
                assert gu.sampled_token_near(ref["logits"][0, i], w.temps[b], ri.u_draft[b, 0, i],
                                             int(tok_np[b, 0, i])), (b, i)
    del lg
    # mixed verify on synthetic inputs: greedy for the first half, T=1 for the rest
    rng = np.random.default_rng(3)
    dtok = rng.integers(0, w.shape.V, size=(w.B, 1, w.shape.K))
    dlog = fs.normal(31, (w.B, 1, w.shape.K, w.shape.V))
    tgt = fs.target_logits(w, r, dtok, dlog)
    h = w.B // 2
    n, br, out = ctx.verify_greedy(to_device(tgt[:h]), to_device(dtok[:h].astype(np.int32)))
    want = gu.verify_oracle_all(tgt[:h], None, dtok[:h], 0, None, None, True)
    np.testing.assert_array_equal(gu.to_np(n), want[0])
    np.testing.assert_array_equal(gu.to_np(out), want[2])
    n, br, out = ctx.verify_sample(to_device(tgt[h:]), to_device(dlog[h:]),
                                   to_device(dtok[h:].astype(np.int32)), 1.0,
                                   to_device(ri.u_accept[h:]), to_device(ri.u_res[h:]))
    (wn, wb, wo), ties = gu.sample_tie_zone(tgt[h:], dlog[h:], dtok[h:], 1.0, ri.u_accept[h:],
                                            ri.u_res[h:])
    ok = ~ties
    np.testing.assert_array_equal(gu.to_np(n)[ok], wn[ok])
    np.testing.assert_array_equal(gu.to_np(out)[ok], wo[ok])
    ctx.close()


# ------------------------------------------------------------------ edge cases (fp32 tiny)
def test_edge_cases_ragged_context_and_slots():
    base = fs.WORKLOADS["tiny_f32"]
    w = dataclasses.replace(base, B=3, n_noise=2, ctx=40)
    ctx = gu.make_ctx(w, max_new=16)
    W = gu.weights64(w.shape, w.dtype)
    hid = {b: fs.prefill_hidden(w, b) for b in range(3)}
    # slot 0: 40 rows in ragged chunks, then rows 5..9 rewritten
    for p0, n in [(0, 16), (16, 16), (32, 8)]:
        ctx.project([0], to_device(hid[0][None, p0:p0 + n]), [p0])
    redo = fs.normal(55, (5, w.shape.n_taps, w.shape.hidden))
    ctx.project([0], to_device(redo[None]), [5])
    rows0 = hid[0].copy()
    rows0[5:10] = redo
    rows0 = rows0[:10]  # the slot's length becomes pos0 + n_new = 10
    # slot 2: 7 rows; slot 1: never projected (context length 0)
    ctx.project([2], to_device(hid[2][None, :7]), [0])
    noise = fs.normal(56, (3, 2, w.shape.K, w.shape.V))
    seqs = [2, 0, 1]
    tok, lg = ctx.draft(seqs, to_device(noise), (0.0, 1.0), [0.0, 0.0, 0.0])
    lg = gu.to_np(lg)
    for q, (slot, rows) in enumerate([(2, hid[2][:7]), (0, rows0), (1, hid[1][:0])]):
        _, kv = om.project_context(W, w.shape.n_blocks, rows)
        ref = om.draft(W, w.shape, kv, noise[q], (0.0, 1.0))
        gu.assert_logits_close(lg[q], ref["logits"], "f32", f"slot {slot}")
    ctx.close()


def test_argument_errors():
    w = fs.WORKLOADS["tiny_f32"]
    ctx = gu.make_ctx(w)
    noise = to_device(fs.round_inputs(w, 0).noise)
    bad = [
        lambda: ctx.draft([0], noise, (0.0, 0.5), [0.0]),            # grid must end at 1
        lambda: ctx.draft([0], noise, (0.0, 0.6, 0.5, 1.0), [0.0]),  # must increase
        lambda: ctx.draft([0], noise, (0.0, 1.0), [1.0]),            # sampling without u
        lambda: ctx.draft([0], noise, (0.0, 1.0), [-1.0]),
        lambda: ctx.draft([5], noise, (0.0, 1.0), [0.0]),            # slot out of range
        lambda: ctx.project([0], to_device(np.zeros((1, 3, 5, 256), np.float32)), [w.ctx + 7]),
        lambda: ctx.project([0, 0], to_device(np.zeros((2, 3, 5, 256), np.float32)), [0, 0]),
    ]
    for f in bad:
        with pytest.raises(FlashmapError) as e:
            f()
        assert e.value.status == FM_ERR_ARG
    ctx.close()


# ------------------------------------------------------------------ factorised drafting
@pytest.mark.parametrize("name,T", [("tiny_f32", 0.0), ("tiny_f32", 0.8)])
def test_factorised_draft_matches_per_position_oracle(name, T):
    # position i from its own noise block: the oracle drafts each block and
    # keeps its position i
    w = dataclasses.replace(fs.WORKLOADS[name], temps=(T,))
    K = w.shape.K
    ctx = gu.make_ctx(dataclasses.replace(w, n_noise=K))
    gu.gpu_prefill(ctx, w, [0])
    kv = gu.oracle_kv(w, 0, None)
    W = gu.weights64(w.shape, w.dtype)
    for r in range(2):
        X = fs.factorised_noise(w, r)
        u = fs.uniform(6000 + r, (1, K))
        tok, lg = ctx.draft_factorised([0], to_device(X, w.dtype), w.t_grid, w.temps,
                                       u_draft=to_device(u) if T > 0 else None)
        tok, lg = gu.to_np(tok)[0], gu.to_np(lg)[0]
        ref = om.draft(W, w.shape, kv, X[0], w.t_grid)
        want_logits = np.stack([ref["logits"][i, i] for i in range(K)])
        gu.assert_logits_close(lg, want_logits, w.dtype, f"round {r}")
        for i in range(K):
            if T == 0:
                if om.margins(want_logits[i]) > gu.MARGIN:
                    assert tok[i] == om.argmax_lowest(want_logits[i]), (r, i)
            else:
                y, sure = gu.sampled_token_sure(want_logits[i], T, u[0, i])
                if sure:
                    assert tok[i] == y, (r, i)
    ctx.close()
