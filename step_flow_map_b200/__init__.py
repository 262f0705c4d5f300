"""ctypes binding of libflashmap_b200.so: the flow-map block drafter and
prefix verifier for B200 (sm_100a).

Argument marshalling only: every step of the draft and the verify runs in
the library's CUDA kernels.  Functions carry the C names declared in
``include/flashmap.h``.  Device buffers may be given as integers (device
addresses) or as objects with ``data_ptr()`` (e.g. torch tensors); streams
as integers, ``None`` (legacy default stream) or objects with
``cuda_stream``.  Importing this package does not need a GPU; loading the
library fails loudly when it has not been built.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libflashmap_b200.so")

FM_OK, FM_ERR_ARG, FM_ERR_CUDA, FM_ERR_OOM, FM_ERR_TIMEOUT, FM_ERR_UNSUPPORTED = 0, -1, -2, -3, -4, -5
FM_F32, FM_BF16 = 0, 1
FM_MAX_CALL_SEQS = 256
FM_MAX_STEPS = 8

EXPORTS = (
    "fm_load_weights", "fm_free", "fm_last_error", "fm_project_context",
    "fm_draft", "fm_verify_greedy", "fm_verify_sample", "fm_profile", "fm_profile_read", "fm_device_status",
    "fm_verify_greedy_noalloc", "fm_draft_factorised", "fm_build_tree", "fm_tree_attention",
    "fm_verify_greedy_tree", "fm_verify_sample_tree", "fm_selftest_exp",
)
FM_PROF = {"embed": 0, "dit_gemm": 1, "attn": 2, "norm": 3, "lm_head": 4, "context": 5,
           "verify": 6, "other": 7}
FM_PROF_N = 8


class FlashmapError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"flashmap status {status}: {msg}")
        self.status = status


class fm_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "V", "d", "n_blocks", "n_heads", "mlp", "K", "target_hidden", "n_taps",
        "dtype", "max_ctx", "max_seqs", "max_noise", "max_new")]


_vp = ctypes.c_void_p
_pvp = ctypes.POINTER(ctypes.c_void_p)


class fm_weights(ctypes.Structure):
    _fields_ = [("E", _vp), ("W_lm", _vp), ("W_fc", _vp), ("W_ts1", _vp), ("W_ts2", _vp),
                ("W_tt1", _vp), ("W_tt2", _vp), ("W_ada_f", _vp), ("W_qkv", _pvp),
                ("W_o", _pvp), ("W_up", _pvp), ("W_down", _pvp), ("W_ada", _pvp)]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load the library once; raise if it is missing (there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise FileNotFoundError(
            f"{path} is missing: build it with `python -m step_flow_map_b200.build` "
            "(no CPU fallback exists)")
    lib = ctypes.CDLL(path)
    i, p, f, st = ctypes.c_int, ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p
    lib.fm_last_error.restype = ctypes.c_char_p
    lib.fm_last_error.argtypes = []
    lib.fm_free.restype = None
    lib.fm_free.argtypes = [p]
    lib.fm_load_weights.restype = i
    lib.fm_load_weights.argtypes = [ctypes.POINTER(p), ctypes.POINTER(fm_config),
                                    ctypes.POINTER(fm_weights), st]
    i32p = ctypes.POINTER(ctypes.c_int32)
    lib.fm_project_context.restype = i
    lib.fm_project_context.argtypes = [p, i32p, i, p, i, i32p, st]
    lib.fm_draft.restype = i
    lib.fm_draft.argtypes = [p, i32p, i, p, i, ctypes.POINTER(f), i, ctypes.POINTER(f), p, p, p, st]
    lib.fm_draft_factorised.restype = i
    lib.fm_draft_factorised.argtypes = [p, i32p, i, p, ctypes.POINTER(f), i, ctypes.POINTER(f), p, p,
                                        p, st]
    lib.fm_build_tree.restype = i
    lib.fm_build_tree.argtypes = [p, i, i, i, p, p, p, p, p, p, st]
    lib.fm_tree_attention.restype = i
    lib.fm_tree_attention.argtypes = [p, p, p, p, p, p, p, i, i, i, i, i, p, st]
    lib.fm_verify_greedy_tree.restype = i
    lib.fm_verify_greedy_tree.argtypes = [p, p, i, p, p, i, i, i, i, p, p, p, st]
    lib.fm_verify_sample_tree.restype = i
    lib.fm_verify_sample_tree.argtypes = [p, p, i, p, p, p, i, i, i, i, f, p, p, p, p, p, st]
    lib.fm_verify_greedy.restype = i
    lib.fm_verify_greedy.argtypes = [p, p, p, i, i, i, i, p, p, p, st]
    lib.fm_verify_sample.restype = i
    lib.fm_verify_sample.argtypes = [p, p, p, p, i, i, i, i, f, p, p, p, p, p, st]
    lib.fm_verify_greedy_noalloc.restype = i
    lib.fm_verify_greedy_noalloc.argtypes = [p, p, i, i, i, i, p, p, p, st]
    lib.fm_device_status.restype = i
    lib.fm_device_status.argtypes = [p, st]
    lib.fm_selftest_exp.restype = i
    lib.fm_selftest_exp.argtypes = [p, p, p, i, st]
    lib.fm_profile.restype = i
    lib.fm_profile.argtypes = [p, i]
    lib.fm_profile_read.restype = i
    lib.fm_profile_read.argtypes = [p, ctypes.POINTER(ctypes.c_double),
                                    ctypes.POINTER(ctypes.c_int64), i]
    _lib = lib
    return lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(status: int):
    if status != FM_OK:
        raise FlashmapError(status, load_library().fm_last_error().decode())


def _i32(values):
    vals = [int(v) for v in values]
    return (ctypes.c_int32 * len(vals))(*vals)


def _f32(values):
    vals = [float(v) for v in values]
    return (ctypes.c_float * len(vals))(*vals)


def fm_last_error() -> str:
    return load_library().fm_last_error().decode()


def fm_load_weights(cfg: dict, weights: dict, stream=None) -> int:
    """Create a context.  ``cfg``: the fm_config fields; ``weights``: device
    buffers named as in fm_weights, per-block ones as ``W_qkv.<l>`` etc."""
    lib = load_library()
    c = fm_config(**{k: int(cfg[k]) for k, _ in fm_config._fields_})
    nb = c.n_blocks
    keep = {}

    def arr(name):
        a = (ctypes.c_void_p * nb)(*[_ptr(weights[f"{name}.{l}"]) for l in range(nb)])
        keep[name] = a
        return ctypes.cast(a, _pvp)

    w = fm_weights(E=_ptr(weights["E"]), W_lm=_ptr(weights["W_lm"]), W_fc=_ptr(weights["W_fc"]),
                   W_ts1=_ptr(weights["W_ts1"]), W_ts2=_ptr(weights["W_ts2"]),
                   W_tt1=_ptr(weights["W_tt1"]), W_tt2=_ptr(weights["W_tt2"]),
                   W_ada_f=_ptr(weights["W_ada_f"]), W_qkv=arr("W_qkv"), W_o=arr("W_o"),
                   W_up=arr("W_up"), W_down=arr("W_down"), W_ada=arr("W_ada"))
    out = ctypes.c_void_p()
    _check(lib.fm_load_weights(ctypes.byref(out), ctypes.byref(c), ctypes.byref(w), _stream(stream)))
    return out.value


def fm_free(ctx: int) -> None:
    load_library().fm_free(ctx)


def fm_project_context(ctx, seq_ids, hidden, n_new, pos0, stream=None) -> None:
    _check(load_library().fm_project_context(ctx, _i32(seq_ids), len(seq_ids), _ptr(hidden),
                                             int(n_new), _i32(pos0), _stream(stream)))


def fm_draft(ctx, seq_ids, noise, n_noise, t_grid, temperature, u_draft, tokens,
             draft_logits=None, stream=None) -> None:
    _check(load_library().fm_draft(ctx, _i32(seq_ids), len(seq_ids), _ptr(noise), int(n_noise),
                                   _f32(t_grid), len(t_grid) - 1, _f32(temperature),
                                   _ptr(u_draft), _ptr(tokens), _ptr(draft_logits),
                                   _stream(stream)))


def fm_draft_factorised(ctx, seq_ids, noise, t_grid, temperature, u_draft, tokens,
                        draft_logits=None, stream=None) -> None:
    """Position i from its own noise block: noise [n_seqs, K, K, V]."""
    _check(load_library().fm_draft_factorised(ctx, _i32(seq_ids), len(seq_ids), _ptr(noise),
                                              _f32(t_grid), len(t_grid) - 1, _f32(temperature),
                                              _ptr(u_draft), _ptr(tokens), _ptr(draft_logits),
                                              _stream(stream)))


def fm_build_tree(draft, B, N, K, node_token, node_parent, node_depth, n_nodes, draft_node,
                  anc_mask, stream=None) -> None:
    _check(load_library().fm_build_tree(_ptr(draft), B, N, K, _ptr(node_token), _ptr(node_parent),
                                        _ptr(node_depth), _ptr(n_nodes), _ptr(draft_node),
                                        _ptr(anc_mask), _stream(stream)))


def fm_tree_attention(q, k_ctx, v_ctx, k_nodes, v_nodes, anc_mask, n_nodes, B, NN, L, n_heads, dh,
                      out, stream=None) -> None:
    _check(load_library().fm_tree_attention(_ptr(q), _ptr(k_ctx), _ptr(v_ctx), _ptr(k_nodes),
                                            _ptr(v_nodes), _ptr(anc_mask), _ptr(n_nodes), B, NN, L,
                                            n_heads, dh, _ptr(out), _stream(stream)))


def fm_verify_greedy_tree(ctx, node_logits, R, draft, draft_node, B, N, K, V, n_acc, branch,
                          out_tokens, stream=None) -> None:
    _check(load_library().fm_verify_greedy_tree(ctx, _ptr(node_logits), R, _ptr(draft),
                                                _ptr(draft_node), B, N, K, V, _ptr(n_acc),
                                                _ptr(branch), _ptr(out_tokens), _stream(stream)))


def fm_verify_sample_tree(ctx, node_logits, R, draft_logits, draft, draft_node, B, N, K, V,
                          temperature, u_accept, u_res, n_acc, branch, out_tokens,
                          stream=None) -> None:
    _check(load_library().fm_verify_sample_tree(ctx, _ptr(node_logits), R, _ptr(draft_logits),
                                                _ptr(draft), _ptr(draft_node), B, N, K, V,
                                                float(temperature), _ptr(u_accept), _ptr(u_res),
                                                _ptr(n_acc), _ptr(branch), _ptr(out_tokens),
                                                _stream(stream)))


def fm_verify_greedy(ctx, target_logits, draft, B, N, K, V, n_acc, branch, out_tokens,
                     stream=None) -> None:
    _check(load_library().fm_verify_greedy(ctx, _ptr(target_logits), _ptr(draft), B, N, K, V,
                                           _ptr(n_acc), _ptr(branch), _ptr(out_tokens),
                                           _stream(stream)))


def fm_verify_sample(ctx, target_logits, draft_logits, draft, B, N, K, V, temperature,
                     u_accept, u_res, n_acc, branch, out_tokens, stream=None) -> None:
    _check(load_library().fm_verify_sample(ctx, _ptr(target_logits), _ptr(draft_logits),
                                           _ptr(draft), B, N, K, V, float(temperature),
                                           _ptr(u_accept), _ptr(u_res), _ptr(n_acc),
                                           _ptr(branch), _ptr(out_tokens), _stream(stream)))


def fm_profile(ctx, mask: int) -> None:
    _check(load_library().fm_profile(ctx, int(mask)))


def fm_profile_read(ctx, reset: bool = False, times: bool = True):
    """(ms per class, launches per class), each a list of FM_PROF_N numbers.

    ``times=False`` reads the launch counts only (ms comes back as None); use
    it while the recorded events have not run yet, e.g. right after a CUDA
    graph capture.
    """
    ms = (ctypes.c_double * FM_PROF_N)() if times else None
    n = (ctypes.c_int64 * FM_PROF_N)()
    _check(load_library().fm_profile_read(ctx, ms, n, int(bool(reset))))
    return (list(ms) if times else None), list(n)


def fm_selftest_exp(e, mine, ref, stream=None) -> None:
    """The verify's fp64 exp (arguments <= 0) and CUDA's exp of fp64 device array e."""
    _check(load_library().fm_selftest_exp(_ptr(e), _ptr(mine), _ptr(ref), e.numel(), _stream(stream)))


def fm_device_status(ctx, stream=None) -> None:
    """Raise FlashmapError(FM_ERR_TIMEOUT) if a kernel's bounded wait gave up."""
    _check(load_library().fm_device_status(ctx, _stream(stream)))


def fm_verify_greedy_noalloc(target_logits, draft, B, N, K, V, n_acc, branch, out_tokens,
                             stream=None) -> None:
    """Greedy verify without a context or any device allocation (see the header)."""
    _check(load_library().fm_verify_greedy_noalloc(_ptr(target_logits), _ptr(draft), B, N, K, V,
                                                   _ptr(n_acc), _ptr(branch), _ptr(out_tokens),
                                                   _stream(stream)))
