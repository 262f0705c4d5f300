"""Host-side marshalling helpers built on torch device memory.

Uploads host arrays into device tensors of the library's storage type and
wraps the C context in a small object.  No step of the draft or verify
runs here.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (FM_BF16, FM_F32, fm_draft, fm_draft_factorised, fm_free, fm_load_weights,
               fm_project_context, fm_verify_greedy, fm_verify_sample)

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}
FM_DTYPE = {"f32": FM_F32, "bf16": FM_BF16}


def to_device(a, dtype: str = "f32", device="cuda") -> torch.Tensor:
    """Host array -> contiguous device tensor of storage type ``dtype``.

    fp64 arrays (uniforms) stay fp64; integer arrays keep their type; other
    floating arrays become ``dtype``.  For bf16 the values must already be
    bf16-representable; the cast is then exact.
    """
    t = torch.from_numpy(np.ascontiguousarray(a))
    if t.dtype == torch.float64:   # uniforms cross the ABI as fp64
        return t.to(device=device).contiguous()
    t = t.to(device=device, dtype=TORCH_DTYPE[dtype] if t.is_floating_point() else t.dtype)
    return t.contiguous()


class Context:
    """A loaded drafter: device weights plus the C context that borrows them."""

    def __init__(self, shape, dtype: str, weights: dict, max_ctx: int, max_seqs: int,
                 max_noise: int, max_new: int, device="cuda", stream=None):
        self.shape, self.dtype = shape, dtype
        self.weights = {k: to_device(v, dtype, device) for k, v in weights.items()}
        cfg = dict(V=shape.V, d=shape.d, n_blocks=shape.n_blocks, n_heads=shape.n_heads,
                   mlp=shape.mlp, K=shape.K, target_hidden=shape.hidden, n_taps=shape.n_taps,
                   dtype=FM_DTYPE[dtype], max_ctx=max_ctx, max_seqs=max_seqs,
                   max_noise=max_noise, max_new=max_new)
        self.cfg = cfg
        self.ctx = fm_load_weights(cfg, self.weights, stream)

    def close(self):
        if self.ctx:
            fm_free(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def project(self, seq_ids, hidden: torch.Tensor, pos0, stream=None):
        n_new = hidden.shape[1]
        fm_project_context(self.ctx, seq_ids, hidden, n_new, pos0, stream)

    def draft(self, seq_ids, noise: torch.Tensor, t_grid, temps, u_draft=None, logits=True,
              stream=None):
        n_seqs, n_noise, K, V = noise.shape
        tokens = torch.empty((n_seqs, n_noise, K), dtype=torch.int32, device=noise.device)
        out_logits = (torch.empty((n_seqs, n_noise, K, V), dtype=torch.float32, device=noise.device)
                      if logits else None)
        fm_draft(self.ctx, seq_ids, noise, n_noise, t_grid, temps, u_draft, tokens, out_logits,
                 stream)
        return tokens, out_logits

    def draft_factorised(self, seq_ids, noise: torch.Tensor, t_grid, temps, u_draft=None,
                         logits=True, stream=None):
        """noise [n_seqs, K, K, V]: position i of each block from noise block i."""
        n_seqs, K, _, V = noise.shape
        tokens = torch.empty((n_seqs, K), dtype=torch.int32, device=noise.device)
        out_logits = (torch.empty((n_seqs, K, V), dtype=torch.float32, device=noise.device)
                      if logits else None)
        fm_draft_factorised(self.ctx, seq_ids, noise, t_grid, temps, u_draft, tokens, out_logits,
                            stream)
        return tokens, out_logits

    def verify_greedy(self, target: torch.Tensor, draft: torch.Tensor, stream=None):
        B, N, K1, V = target.shape
        dev = target.device
        n = torch.empty(B, dtype=torch.int32, device=dev)
        br = torch.empty(B, dtype=torch.int32, device=dev)
        out = torch.empty((B, K1), dtype=torch.int32, device=dev)
        fm_verify_greedy(self.ctx, target, draft, B, N, K1 - 1, V, n, br, out, stream)
        return n, br, out

    def verify_sample(self, target, draft_logits, draft, T, u_accept, u_res, stream=None):
        B, N, K1, V = target.shape
        dev = target.device
        n = torch.empty(B, dtype=torch.int32, device=dev)
        br = torch.empty(B, dtype=torch.int32, device=dev)
        out = torch.empty((B, K1), dtype=torch.int32, device=dev)
        fm_verify_sample(self.ctx, target, draft_logits, draft, B, N, K1 - 1, V, T, u_accept,
                         u_res, n, br, out, stream)
        return n, br, out
