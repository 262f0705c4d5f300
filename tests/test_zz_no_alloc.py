"""Greedy verify that allocates nothing (fm_verify_greedy_noalloc).

Callers that cannot allocate device memory -- a server whose memory arena
owns the whole GPU, or a verify-only user without a drafter context -- use
this entry point; its scratch is a fixed device array inside the library.
This file runs last so that a failure here comes after every other test.
"""
import dataclasses

import numpy as np
import pytest
import torch

import fm_synth as fs
from step_flow_map_b200 import fm_verify_greedy_noalloc
from step_flow_map_b200.host import to_device

import gpu_util as gu

pytestmark = pytest.mark.gpu


def _case(B, N, seed, V=151936, K=16):
    w = dataclasses.replace(fs.WORKLOADS["tiny_f32"], B=B, n_noise=N, ctx=4, new_rows=1,
                            target="near_draft", target_std=1.5,
                            shape=dataclasses.replace(fs.TINY, V=V, K=K))
    rng = np.random.default_rng(seed)
    tok = rng.integers(0, V, size=(B, N, K))
    for b in range(B):
        for j in range(1, N):
            cut = int(rng.integers(0, K + 1))
            tok[b, j, :cut] = tok[b, 0, :cut]
    tgt = fs.target_logits(w, seed, tok)
    return w, to_device(tgt), to_device(tok.astype(np.int32))


def _noalloc(tgt, tok):
    B, N, K1, V = tgt.shape
    n = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    br = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    out = torch.full((B, K1), -7, dtype=torch.int32, device="cuda")
    fm_verify_greedy_noalloc(tgt, tok, B, N, K1 - 1, V, n, br, out,
                             torch.cuda.current_stream())
    torch.cuda.synchronize()
    return gu.to_np(n), gu.to_np(br), gu.to_np(out)


def test_noalloc_matches_context_verify_twice():
    assert torch.cuda.is_available()
    w1, tgt1, tok1 = _case(B=5, N=2, seed=71)
    w2, tgt2, tok2 = _case(B=3, N=4, seed=72)
    # the existing entry point, through a context
    ctx = gu.make_ctx(dataclasses.replace(w1, B=5, n_noise=4), max_new=4)
    want1 = [gu.to_np(t) for t in ctx.verify_greedy(tgt1, tok1)]
    want2 = [gu.to_np(t) for t in ctx.verify_greedy(tgt2, tok2)]
    ctx.close()
    # two calls in a row share the library's scratch
    got1 = _noalloc(tgt1, tok1)
    got2 = _noalloc(tgt2, tok2)
    for got, want in ((got1, want1), (got2, want2)):
        for g, wv in zip(got, want):
            np.testing.assert_array_equal(g, wv)
    assert want1[0].max() > 0 and want2[0].max() > 0
    # and both against the fp64 oracle's greedy verify directly
    for got, tgt, tok in ((got1, tgt1, tok1), (got2, tgt2, tok2)):
        ref = gu.verify_oracle_all(gu.to_np(tgt), None, gu.to_np(tok), 0, None, None, True)
        for g, wv in zip(got, ref):
            np.testing.assert_array_equal(g, wv)


def test_noalloc_nan_and_ties_match_the_oracle():
    # NaN never wins (it ranks below -inf), ties go to the lowest index, a
    # row of NaN gives token 0
    B, N, K, V = 2, 1, 16, 4099
    tgt = np.zeros((B, N, K + 1, V), np.float32)
    tok = np.zeros((B, N, K), np.int64)
    tgt[0, 0, :, 7] = 1.0
    tok[0, 0, :] = 7
    tgt[0, 0, 3, 7] = np.nan                 # row 3: 7 is NaN, so the argmax is the lowest tie 0
    tgt[1, 0, 0, :] = np.nan                 # a row of NaN -> token 0
    tgt[1, 0, 1, :] = -np.inf
    tgt[1, 0, 1, :5] = np.nan                # NaN below -inf: the argmax is 5
    tok[1, 0, 1] = 5
    got = _noalloc(to_device(tgt), to_device(tok.astype(np.int32)))
    ref = gu.verify_oracle_all(tgt, None, tok, 0, None, None, True)
    for g, wv in zip(got, ref):
        np.testing.assert_array_equal(g, wv)
    assert list(ref[0]) == [3, 16]


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from step_flow_map_b200 import FM_ERR_UNSUPPORTED, FlashmapError
    tgt = torch.zeros((1, 1, 17, 8), dtype=torch.float32, device="cuda")
    tok = torch.zeros((1, 1, 16), dtype=torch.int32, device="cuda")
    o = torch.zeros(4096, dtype=torch.int32, device="cuda")
    # every limit is checked on the host, before anything is queued
    for B, N, K, V in ((2000, 1, 16, 8),          # more than 1024 sequences
                       (1, 64, 16, 8),            # N*(K+1) = 1088 rows per sequence
                       (1024, 2, 16, 8),          # B*N*(K+1) = 34816 rows
                       (1, 1, 2**31 - 1, 8),      # K so large that N*(K+1) would wrap
                       (1, 2**31 - 1, 16, 8),
                       (1, 1, 16, 2**30)):        # V beyond 2^28
        with pytest.raises(FlashmapError) as e:
            fm_verify_greedy_noalloc(tgt, tok, B, N, K, V, o, o, o)
        assert e.value.status == FM_ERR_UNSUPPORTED, (B, N, K, V)
