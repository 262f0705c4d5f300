"""Tensor-core (tcgen05) GEMM path on a small bf16 drafter, against the oracle.

Runs before the full-size tests: every GEMM of the draft (context fc and
keys/values, x.E with split-K, QKV/O/MLP, LM head with stored logits and
with the fused argmax) goes through the tensor-core kernel at several
activation-row counts (BN = 16, 64, 256 with a ragged tail).
"""
import dataclasses
import os

import numpy as np
import pytest
import torch

import fm_synth as fs
from oracle import flashmap as om
from step_flow_map_b200 import fm_device_status
from step_flow_map_b200.host import Context, to_device

import gpu_util as gu

pytestmark = pytest.mark.gpu

SMALL = fs.Shape(V=1024, d=128, n_blocks=2, n_heads=1, mlp=256, K=16, hidden=64)


def _workload(B, N, t_grid=(0.0, 1.0), temps=None, ctx=40):
    return dataclasses.replace(fs.WORKLOADS["qwen3_8b_bs1"], name="small_bf16", shape=SMALL,
                               B=B, n_noise=N, ctx=ctx, new_rows=17, t_grid=t_grid,
                               temps=temps or tuple([0.0] * B))


def _run(w, env_off=False, logits=True, no_persistent=False, no_cluster=False):
    if env_off:
        os.environ["FM_DISABLE_TC"] = "1"
    if no_persistent:
        os.environ["FM_DISABLE_PERSISTENT"] = "1"
    if no_cluster:
        os.environ["FM_DISABLE_TC_CLUSTER"] = "1"
    try:
        ctx = gu.make_ctx(w, max_new=64)
    finally:
        os.environ.pop("FM_DISABLE_TC", None)
        os.environ.pop("FM_DISABLE_PERSISTENT", None)
        os.environ.pop("FM_DISABLE_TC_CLUSTER", None)
    seqs = list(range(w.B))
    gu.gpu_prefill(ctx, w, seqs, max_new=64)
    gu.gpu_new_rows(ctx, w, 0, seqs)
    ri = fs.round_inputs(w, 0)
    tok, lg = ctx.draft(seqs, to_device(ri.noise, "bf16"), w.t_grid, w.temps,
                        u_draft=to_device(ri.u_draft), logits=logits)
    torch.cuda.synchronize()
    fm_device_status(ctx.ctx)
    out = (gu.to_np(tok), None if lg is None else gu.to_np(lg))
    ctx.close()
    return out, ri


@pytest.mark.parametrize("B,N", [(1, 1), (1, 4), (9, 2)])
def test_tc_draft_matches_oracle(B, N):
    w = _workload(B, N)
    (tok, lg), ri = _run(w)
    for b in sorted({0, B - 1}):
        ref = gu.oracle_draft(w, b, 0)
        gu.assert_logits_close(lg[b], ref["logits"], "bf16", f"seq {b}")
        gu.assert_tokens_on_margin(tok[b], ref["logits"], f"seq {b}")
    # the fused LM-head argmax (no logits written) picks the same tokens
    (tok2, none), _ = _run(w, logits=False)
    assert none is None
    np.testing.assert_array_equal(tok2, tok)


def test_persistent_pass_matches_per_kernel_path():
    # one sequence, one noise draft: the persistent DiT pass (with the 17 new
    # context rows projected inside its QKV phases) against one kernel per GEMM
    w = _workload(1, 1)
    (tok_p, lg_p), _ = _run(w)
    (tok_k, lg_k), _ = _run(w, no_persistent=True)
    np.testing.assert_allclose(lg_p, lg_k, atol=2e-2, rtol=1e-2)
    ref = gu.oracle_draft(w, 0, 0)
    gu.assert_logits_close(lg_p[0], ref["logits"], "bf16", "persistent")


def test_persistent_pass_context_rows_reach_the_cache():
    # round 0 appends 17 rows (projected inside the first draft's QKV phases);
    # round 1 appends 17 more after them and drafts against all of them, so
    # its logits check the keys/values the first pass wrote
    w = _workload(1, 1)
    ctx = Context(w.shape, w.dtype, gu.weights(w.shape, w.dtype), max_ctx=w.ctx + 40,
                  max_seqs=1, max_noise=1, max_new=64)
    gu.gpu_prefill(ctx, w, [0], max_new=64)
    rows = [fs.prefill_hidden(w, 0)]
    for r, p0 in ((0, w.ctx), (1, w.ctx + 17)):
        ri = fs.round_inputs(w, r)
        ctx.project([0], to_device(ri.new_hidden, "bf16"), [p0])
        rows.append(ri.new_hidden[0])
        tok, lg = ctx.draft([0], to_device(ri.noise, "bf16"), w.t_grid, w.temps)
        torch.cuda.synchronize()
        fm_device_status(ctx.ctx)
        W = gu.weights64(w.shape, w.dtype)
        _, kv = om.project_context(W, w.shape.n_blocks, np.concatenate(rows, axis=0))
        ref = om.draft(W, w.shape, kv, ri.noise[0], w.t_grid)
        gu.assert_logits_close(gu.to_np(lg)[0], ref["logits"], "bf16", f"round {r}")
    ctx.close()


def test_cluster_splitk_matches_global_reduction():
    # four noise drafts of one sequence: 64 activation rows, one activation
    # tile, so the split-K GEMMs of the draft (x.E in 8 splits, QKV, O and
    # the MLP) sum their partial tiles inside a thread-block cluster through
    # distributed shared memory; the same draft with the partials reduced
    # through global memory (other split counts) agrees to rounding, and
    # both match the oracle
    w = _workload(1, 4)
    (tok_c, lg_c), _ = _run(w)
    (tok_g, lg_g), _ = _run(w, no_cluster=True)
    np.testing.assert_allclose(lg_c, lg_g, atol=2e-2, rtol=1e-2)
    ref = gu.oracle_draft(w, 0, 0)
    gu.assert_logits_close(lg_c[0], ref["logits"], "bf16", "cluster")
    gu.assert_logits_close(lg_g[0], ref["logits"], "bf16", "global")


def test_tc_matches_cuda_core_path():
    w = _workload(2, 1)
    (tok_tc, lg_tc), _ = _run(w)
    (tok_cc, lg_cc), _ = _run(w, env_off=True)
    np.testing.assert_allclose(lg_tc, lg_cc, atol=2e-2, rtol=1e-2)


def test_tc_two_step():
    w = _workload(1, 2, t_grid=(0.0, 0.5, 1.0), temps=(1.0,))
    (tok, lg), ri = _run(w)
    ref = gu.oracle_draft(w, 0, 0)
    gu.assert_logits_close(lg[0], ref["logits"], "bf16", "two-step")
    for j in range(w.n_noise):
        for i in range(w.shape.K):
            y, sure = gu.sampled_token_sure(ref["logits"][j, i], 1.0, ri.u_draft[0, j, i])
            if sure:
                assert tok[0, j, i] == y


def test_nan_logit_never_wins():
    # a NaN row of the LM head makes one token's logit NaN in every row; the
    # fused LM-head argmax (no logits written) and the stored-logits path
    # must both skip it, as the oracle's argmax does
    w = _workload(1, 1)
    ref0 = gu.oracle_draft(w, 0, 0)
    vstar = int(np.argmax(ref0["logits"][0, 0]))
    W = {k: v.copy() for k, v in gu.weights(w.shape, w.dtype).items()}
    W["W_lm"][vstar] = np.nan
    W64 = {k: v.astype(np.float64) for k, v in W.items()}
    rows = np.concatenate([fs.prefill_hidden(w, 0), fs.round_inputs(w, 0).new_hidden[0]], axis=0)
    _, kv = om.project_context(W64, w.shape.n_blocks, rows)
    refs = [om.draft(W64, w.shape, kv, fs.round_inputs(w, r).noise[0], w.t_grid) for r in range(4)]
    checked = 0
    for logits in (False, True):
        ctx = Context(w.shape, w.dtype, W, max_ctx=w.ctx + 40, max_seqs=1, max_noise=1, max_new=64)
        gu.gpu_prefill(ctx, w, [0], max_new=64)
        gu.gpu_new_rows(ctx, w, 0, [0])
        for r, ref in enumerate(refs):
            ri = fs.round_inputs(w, r)
            assert (ref["tokens"] != vstar).all()
            tok, _ = ctx.draft([0], to_device(ri.noise, "bf16"), w.t_grid, w.temps, logits=logits)
            torch.cuda.synchronize()
            fm_device_status(ctx.ctx)
            got = gu.to_np(tok)[0]
            assert (got != vstar).all(), (logits, r)
            clean = np.where(np.isnan(ref["logits"]), -np.inf, ref["logits"])
            sure = om.margins(clean) > gu.MARGIN
            np.testing.assert_array_equal(got[sure], ref["tokens"][sure])
            checked += int(sure.sum())
        ctx.close()
    assert checked >= 4
