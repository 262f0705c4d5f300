"""Failure detection on the GPU without a fault: a bounded wait runs out.

Every wait inside the kernels is bounded (about two seconds).  The test hook
FM_TEST_STALL=1, read when a context is created, makes the next persistent
DiT pass wait for a handoff word that no phase writes, so that wait -- and
every wait of the other CTAs, which read the abort word while they poll --
gives up.  The pass then stops early, fm_device_status reports
FM_ERR_TIMEOUT once, and the same context drafts correctly afterwards (the
round's context rows are projected again, as a caller does after a failed
round).  Nothing here traps, faults or waits without a bound.
"""
import dataclasses
import os
import time

import numpy as np
import pytest
import torch

import fm_synth as fs
from oracle import flashmap as om
from step_flow_map_b200 import FM_ERR_TIMEOUT, FlashmapError, fm_device_status
from step_flow_map_b200.host import Context, to_device

import gpu_util as gu

pytestmark = pytest.mark.gpu

SMALL = fs.Shape(V=1024, d=128, n_blocks=2, n_heads=1, mlp=256, K=16, hidden=64)


def test_bounded_wait_runs_out_and_the_context_recovers():
    assert torch.cuda.is_available()
    w = dataclasses.replace(fs.WORKLOADS["qwen3_8b_bs1"], name="small_bf16", shape=SMALL, ctx=40)
    W = gu.weights(w.shape, w.dtype)
    os.environ["FM_TEST_STALL"] = "1"
    try:
        ctx = Context(w.shape, w.dtype, W, max_ctx=w.ctx + 24, max_seqs=1, max_noise=1, max_new=64)
    finally:
        os.environ.pop("FM_TEST_STALL", None)
    ctx.project([0], to_device(fs.prefill_hidden(w, 0)[None], "bf16"), [0])
    ri = fs.round_inputs(w, 0)
    new_rows = to_device(ri.new_hidden, "bf16")
    ctx.project([0], new_rows, [w.ctx])
    noise = to_device(ri.noise, "bf16")
    torch.cuda.synchronize()
    t0 = time.time()
    ctx.draft([0], noise, w.t_grid, w.temps)
    torch.cuda.synchronize()
    waited = time.time() - t0
    with pytest.raises(FlashmapError) as e:
        fm_device_status(ctx.ctx)
    assert e.value.status == FM_ERR_TIMEOUT
    assert waited < 60
    fm_device_status(ctx.ctx)            # reported once, then clear
    # the same context: project the round's rows again and draft
    ctx.project([0], new_rows, [w.ctx])
    tok, lg = ctx.draft([0], noise, w.t_grid, w.temps)
    torch.cuda.synchronize()
    fm_device_status(ctx.ctx)
    W64 = gu.weights64(w.shape, w.dtype)
    rows = np.concatenate([fs.prefill_hidden(w, 0), ri.new_hidden[0]], axis=0)
    _, kv = om.project_context(W64, w.shape.n_blocks, rows)
    ref = om.draft(W64, w.shape, kv, ri.noise[0], w.t_grid)
    gu.assert_logits_close(gu.to_np(lg)[0], ref["logits"], "bf16", "after recovery")
    gu.assert_tokens_on_margin(gu.to_np(tok)[0], ref["logits"], "after recovery")
    ctx.close()
