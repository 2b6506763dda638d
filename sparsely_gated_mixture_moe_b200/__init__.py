"""Python binding of libmoe: the sparsely-gated Mixture-of-Experts layer forward on B200.

A thin ctypes layer over the C ABI in include/moe.h.  Every step of the layer runs in
the library's CUDA kernels; this module only marshals arguments (device pointers of
torch tensors, the stream handle, the config struct) and turns status codes into
exceptions.  There is no CPU fallback: importing fails loudly when libmoe.so has not
been built, and every call requires CUDA tensors.

    python sparsely_gated_mixture_moe_b200/build_lib.py      # build libmoe.so in-tree
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from .config import (ACT, DEVERR, DTYPE, GATING, MoEConfig, MoEError, STATUS, make_config)

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe.so")


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            "libmoe.so is not built (expected at %s); build it with "
            "`python sparsely_gated_mixture_moe_b200/build_lib.py`" % _LIB_PATH)
    lib = ctypes.CDLL(_LIB_PATH)
    P = ctypes.c_void_p
    C = ctypes.POINTER(MoEConfig)
    sig = {
        "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "moe_capacity": (ctypes.c_int64, [C]),
        "moe_workspace_size": (ctypes.c_size_t, [C]),
        "moe_forward_workspace_size": (ctypes.c_size_t, [C]),
        "moe_route": (ctypes.c_int, [C, P, P, P, P, P, P, P, P, P, P, P, P]),
        "moe_permute": (ctypes.c_int, [C, P, P, P, P, P, P, P, P, P]),
        "moe_expert_ffn": (ctypes.c_int, [C, P, P, P, P, P, P, P, P]),
        "moe_combine": (ctypes.c_int, [C, P, P, P, P, P, P]),
        "moe_expert_ffn_combine": (ctypes.c_int, [C, P, P, P, P, P, P, P, P, P, P, P]),
        "moe_expert_ffn_gather": (ctypes.c_int, [C, P, P, P, P, P, P, P, P, P]),
        "moe_expert_ffn_combine_gather": (ctypes.c_int, [C, P, P, P, P, P, P, P, P, P, P, P]),
        "moe_forward": (ctypes.c_int, [C, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P]),
        "moe_get_error": (ctypes.c_int, [P, P, ctypes.POINTER(ctypes.c_int32)]),
        "moe_last_launch_count": (ctypes.c_int32, []),
        "moe_bf16_to_f16": (ctypes.c_int, [P, P, ctypes.c_int64, P, P]),
        "moe_permute_noalloc": (ctypes.c_int, [C, P, P, P, P, P, P, P, P]),
        "moe_erf_check": (ctypes.c_int, [P, P, P, ctypes.c_int64, P]),
        "moe_gelu_check": (ctypes.c_int, [P, P, P, ctypes.c_int64, P]),
        "moe_expert_ffn_grouped": (ctypes.c_int, [C, P, ctypes.c_int64, P, ctypes.c_int32, P, P, P, P,
                                                  P, P]),
        "moe_train_state_size": (ctypes.c_size_t, [C]),
        "moe_backward_workspace_size": (ctypes.c_size_t, [C]),
        "moe_forward_train": (ctypes.c_int, [C] + [P] * 17),
        "moe_backward": (ctypes.c_int, [C] + [P] * 13 + [ctypes.c_float, ctypes.c_float] +
                         [P] * 10),
        "moe_wait_timeout_check": (ctypes.c_int, [P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()
LIB_PATH = _LIB_PATH


def _ptr(t: Optional[torch.Tensor], what: str):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % what)
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor (libmoe has no CPU path)" % what)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % what)
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, what: str):
    if status != 0:
        raise MoEError(status, "%s: %s" % (what, lib.moe_status_string(status).decode()))


def moe_capacity(cfg: MoEConfig) -> int:
    """C = ceil(cf*T*k/E) computed by the library (-1: no limit)."""
    return int(lib.moe_capacity(ctypes.byref(cfg)))


def moe_workspace_size(cfg: MoEConfig) -> int:
    return int(lib.moe_workspace_size(ctypes.byref(cfg)))


def moe_forward_workspace_size(cfg: MoEConfig) -> int:
    return int(lib.moe_forward_workspace_size(ctypes.byref(cfg)))


def workspace(cfg: MoEConfig, device="cuda", forward: bool = False) -> torch.Tensor:
    """A zero-filled device workspace of the size the library asks for."""
    n = moe_forward_workspace_size(cfg) if forward else moe_workspace_size(cfg)
    if n == 0:
        raise MoEError(2, "config is invalid or unsupported")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def moe_route(cfg, x, w_gate, topk_idx, topk_gate, ws, w_noise=None, noise=None,
              logit_bias=None, importance=None, load=None, near_tie=None, stream=None):
    _check(lib.moe_route(ctypes.byref(cfg), _ptr(x, "x"), _ptr(w_gate, "w_gate"),
                         _ptr(w_noise, "w_noise"), _ptr(noise, "noise"),
                         _ptr(logit_bias, "logit_bias"), _ptr(topk_idx, "topk_idx"),
                         _ptr(topk_gate, "topk_gate"), _ptr(importance, "importance"),
                         _ptr(load, "load"), _ptr(near_tie, "near_tie"), _ptr(ws, "ws"),
                         _stream(stream)), "moe_route")


def moe_permute(cfg, topk_idx, x, counts, offsets, perm_src, slot_pos, x_perm, ws, stream=None):
    """x_perm (and x) may be None: only the index arrays are written."""
    _check(lib.moe_permute(ctypes.byref(cfg), _ptr(topk_idx, "topk_idx"), _ptr(x, "x"),
                           _ptr(counts, "counts"), _ptr(offsets, "offsets"),
                           _ptr(perm_src, "perm_src"), _ptr(slot_pos, "slot_pos"),
                           _ptr(x_perm, "x_perm"), _ptr(ws, "ws"), _stream(stream)),
           "moe_permute")


def moe_permute_noalloc(cfg, topk_idx, x, counts, offsets, perm_src, slot_pos, x_perm,
                        stream=None):
    """moe_permute with the library's fixed device scratch instead of a workspace (for
    callers that cannot allocate); see include/moe.h for its size limit and sharing."""
    _check(lib.moe_permute_noalloc(ctypes.byref(cfg), _ptr(topk_idx, "topk_idx"), _ptr(x, "x"),
                                   _ptr(counts, "counts"), _ptr(offsets, "offsets"),
                                   _ptr(perm_src, "perm_src"), _ptr(slot_pos, "slot_pos"),
                                   _ptr(x_perm, "x_perm"), _stream(stream)),
           "moe_permute_noalloc")


def moe_expert_ffn(cfg, x_perm, offsets, w1, w2, h, y_perm, ws, stream=None):
    _check(lib.moe_expert_ffn(ctypes.byref(cfg), _ptr(x_perm, "x_perm"), _ptr(offsets, "offsets"),
                              _ptr(w1, "w1"), _ptr(w2, "w2"), _ptr(h, "h"),
                              _ptr(y_perm, "y_perm"), _ptr(ws, "ws"), _stream(stream)),
           "moe_expert_ffn")


def moe_expert_ffn_grouped(cfg, x_rows, offsets, groups, w1, w2, h, y_rows, ws, stream=None):
    """moe_expert_ffn over `groups` row groups, group g running expert g % cfg.E (the rows
    an expert-parallel rank receives, source by source); x_rows' first dimension is the
    row capacity."""
    _check(lib.moe_expert_ffn_grouped(ctypes.byref(cfg), _ptr(x_rows, "x_rows"),
                                      int(x_rows.shape[0]), _ptr(offsets, "offsets"), int(groups),
                                      _ptr(w1, "w1"), _ptr(w2, "w2"), _ptr(h, "h"),
                                      _ptr(y_rows, "y_rows"), _ptr(ws, "ws"), _stream(stream)),
           "moe_expert_ffn_grouped")


def moe_expert_ffn_gather(cfg, x, perm_src, offsets, w1, w2, h, y_perm, ws, stream=None):
    """moe_expert_ffn with permuted row s gathered from x[perm_src[s] // k] by the kernel."""
    _check(lib.moe_expert_ffn_gather(ctypes.byref(cfg), _ptr(x, "x"), _ptr(perm_src, "perm_src"),
                                     _ptr(offsets, "offsets"), _ptr(w1, "w1"), _ptr(w2, "w2"),
                                     _ptr(h, "h"), _ptr(y_perm, "y_perm"), _ptr(ws, "ws"),
                                     _stream(stream)), "moe_expert_ffn_gather")


def moe_expert_ffn_combine_gather(cfg, x, offsets, perm_src, slot_pos, topk_gate, w1, w2, h, y,
                                  ws, stream=None):
    """moe_expert_ffn_combine with the permuted rows gathered from x."""
    _check(lib.moe_expert_ffn_combine_gather(
        ctypes.byref(cfg), _ptr(x, "x"), _ptr(offsets, "offsets"), _ptr(perm_src, "perm_src"),
        _ptr(slot_pos, "slot_pos"), _ptr(topk_gate, "topk_gate"), _ptr(w1, "w1"), _ptr(w2, "w2"),
        _ptr(h, "h"), _ptr(y, "y"), _ptr(ws, "ws"), _stream(stream)),
        "moe_expert_ffn_combine_gather")


def moe_combine(cfg, y_perm, slot_pos, topk_gate, y, ws, stream=None):
    _check(lib.moe_combine(ctypes.byref(cfg), _ptr(y_perm, "y_perm"), _ptr(slot_pos, "slot_pos"),
                           _ptr(topk_gate, "topk_gate"), _ptr(y, "y"), _ptr(ws, "ws"),
                           _stream(stream)), "moe_combine")


def moe_expert_ffn_combine(cfg, x_perm, offsets, perm_src, slot_pos, topk_gate, w1, w2, h, y,
                           ws, stream=None):
    """moe_expert_ffn + moe_combine as one step (bf16; k = 1, or k = 2 with an fp32 y): the
    down-projection puts gate * row straight into y at its token (a store for k = 1, an
    in-memory add onto the row the up-projection zeroed for k = 2)."""
    _check(lib.moe_expert_ffn_combine(ctypes.byref(cfg), _ptr(x_perm, "x_perm"),
                                      _ptr(offsets, "offsets"), _ptr(perm_src, "perm_src"),
                                      _ptr(slot_pos, "slot_pos"), _ptr(topk_gate, "topk_gate"),
                                      _ptr(w1, "w1"), _ptr(w2, "w2"), _ptr(h, "h"), _ptr(y, "y"),
                                      _ptr(ws, "ws"), _stream(stream)), "moe_expert_ffn_combine")


def fused_combine(cfg) -> bool:
    """Whether moe_expert_ffn_combine applies: bf16 with top-1 routing, or top-2 with an
    fp32 layer output."""
    return cfg.dtype == DTYPE["bf16"] and (cfg.k == 1 or (cfg.k == 2 and not cfg.y_bf16))


def moe_forward(cfg, x, w_gate, w1, w2, y, topk_idx, topk_gate, counts, ws, w_noise=None,
                noise=None, logit_bias=None, importance=None, load=None, near_tie=None,
                stream=None):
    _check(lib.moe_forward(ctypes.byref(cfg), _ptr(x, "x"), _ptr(w_gate, "w_gate"),
                           _ptr(w_noise, "w_noise"), _ptr(noise, "noise"),
                           _ptr(logit_bias, "logit_bias"), _ptr(w1, "w1"), _ptr(w2, "w2"),
                           _ptr(y, "y"), _ptr(topk_idx, "topk_idx"), _ptr(topk_gate, "topk_gate"),
                           _ptr(counts, "counts"), _ptr(importance, "importance"),
                           _ptr(load, "load"), _ptr(near_tie, "near_tie"), _ptr(ws, "ws"),
                           _stream(stream)), "moe_forward")


def train_state(cfg, device="cuda") -> torch.Tensor:
    """A device buffer for the forward state moe_forward_train keeps for moe_backward."""
    n = int(lib.moe_train_state_size(ctypes.byref(cfg)))
    if n == 0:
        raise MoEError(2, "config unsupported by the training path")
    return torch.empty(n, dtype=torch.uint8, device=device)


def backward_workspace(cfg, device="cuda") -> torch.Tensor:
    """A zero-filled device workspace for moe_backward (its error word included)."""
    n = int(lib.moe_backward_workspace_size(ctypes.byref(cfg)))
    if n == 0:
        raise MoEError(2, "config unsupported by the training path")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def moe_forward_train(cfg, x, w_gate, w1, w2, y, topk_idx, topk_gate, counts, state, ws,
                      w_noise=None, noise=None, logit_bias=None, importance=None, load=None,
                      near_tie=None, stream=None):
    _check(lib.moe_forward_train(ctypes.byref(cfg), _ptr(x, "x"), _ptr(w_gate, "w_gate"),
                                 _ptr(w_noise, "w_noise"), _ptr(noise, "noise"),
                                 _ptr(logit_bias, "logit_bias"), _ptr(w1, "w1"), _ptr(w2, "w2"),
                                 _ptr(y, "y"), _ptr(topk_idx, "topk_idx"),
                                 _ptr(topk_gate, "topk_gate"), _ptr(counts, "counts"),
                                 _ptr(importance, "importance"), _ptr(load, "load"),
                                 _ptr(near_tie, "near_tie"), _ptr(state, "state"), _ptr(ws, "ws"),
                                 _stream(stream)), "moe_forward_train")


def moe_backward(cfg, x, w_gate, w1, w2, topk_idx, topk_gate, state, dy, dx, dw_gate, dw1, dw2,
                 dgates, ws, w_noise=None, noise=None, logit_bias=None, importance=None,
                 load=None, w_importance=0.0, w_load=0.0, dw_noise=None, dlogit_bias=None,
                 losses=None, stream=None):
    _check(lib.moe_backward(ctypes.byref(cfg), _ptr(x, "x"), _ptr(w_gate, "w_gate"),
                            _ptr(w_noise, "w_noise"), _ptr(noise, "noise"),
                            _ptr(logit_bias, "logit_bias"), _ptr(w1, "w1"), _ptr(w2, "w2"),
                            _ptr(topk_idx, "topk_idx"), _ptr(topk_gate, "topk_gate"),
                            _ptr(importance, "importance"), _ptr(load, "load"),
                            _ptr(state, "state"), _ptr(dy, "dy"), float(w_importance),
                            float(w_load), _ptr(dx, "dx"), _ptr(dw_gate, "dw_gate"),
                            _ptr(dw_noise, "dw_noise"), _ptr(dlogit_bias, "dlogit_bias"),
                            _ptr(dw1, "dw1"), _ptr(dw2, "dw2"), _ptr(dgates, "dgates"),
                            _ptr(losses, "losses"), _ptr(ws, "ws"), _stream(stream)),
           "moe_backward")


def moe_get_error(ws: torch.Tensor, stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error word."""
    v = ctypes.c_int32(0)
    st = lib.moe_get_error(_ptr(ws, "ws"), _stream(stream), ctypes.byref(v))
    if st not in (0, 4):
        _check(st, "moe_get_error")
    return int(v.value)


def moe_bf16_to_f16(src: torch.Tensor, dst: torch.Tensor, n_inexact=None, stream=None):
    """Re-encode a bf16 CUDA tensor as fp16 into `dst` (same shape); `n_inexact` (an int32
    CUDA tensor of one element, or None) is incremented by the values not kept exactly."""
    if src.dtype != torch.bfloat16 or dst.dtype != torch.float16 or src.shape != dst.shape:
        raise ValueError("moe_bf16_to_f16 needs a bf16 source and an fp16 destination of one shape")
    _check(lib.moe_bf16_to_f16(_ptr(src, "src"), _ptr(dst, "dst"), src.numel(),
                               _ptr(n_inexact, "n_inexact"), _stream(stream)), "moe_bf16_to_f16")


def prepare_weights(cfg: MoEConfig, weights: dict, stream=None) -> dict:
    """Weights as the forward pass takes them: with cfg.hidden_f16, w2 re-encoded to fp16
    by the library (the other tensors are passed through)."""
    out = dict(weights)
    if cfg.hidden_f16 and cfg.dtype == DTYPE["bf16"] and weights["w2"].dtype == torch.bfloat16:
        w2 = torch.empty(weights["w2"].shape, dtype=torch.float16, device=weights["w2"].device)
        moe_bf16_to_f16(weights["w2"], w2, stream=stream)
        out["w2"] = w2
    return out


def last_launch_count() -> int:
    """Kernels queued by the most recent successful call on this thread."""
    return int(lib.moe_last_launch_count())


class MoELayer:
    """Owns the device buffers of one layer configuration and runs its forward pass.

    weights: dict with w_gate [E,d], w1 [E,f,d], w2 [E,d,f] (and w_noise [E,d] for noisy
    gating, logit_bias [E] fp32 if used), CUDA tensors in the config's dtype.  The layer
    output y [T, d] is fp32, or bf16 when the config asks for it (y_bf16).
    """

    def __init__(self, cfg: MoEConfig, weights: dict, device="cuda"):
        self.cfg = cfg
        self.w = prepare_weights(cfg, weights)
        T, k, E, d = cfg.T, cfg.k, cfg.E, cfg.d_model
        self.y = torch.empty(T, d, dtype=torch.bfloat16 if cfg.y_bf16 else torch.float32,
                             device=device)
        self.topk_idx = torch.empty(T, k, dtype=torch.int32, device=device)
        self.topk_gate = torch.empty(T, k, dtype=torch.float32, device=device)
        self.counts = torch.empty(E, dtype=torch.int32, device=device)
        noisy = cfg.gating == GATING["noisy_topk"]
        self.importance = torch.empty(E, dtype=torch.float32, device=device) if noisy else None
        self.load = torch.empty(E, dtype=torch.float32, device=device) if noisy and k < E else None
        self.near_tie = torch.empty(T, dtype=torch.uint8, device=device)
        self.ws = workspace(cfg, device, forward=True)

    def forward(self, x: torch.Tensor, noise: Optional[torch.Tensor] = None, stream=None):
        w = self.w
        moe_forward(self.cfg, x, w["w_gate"], w["w1"], w["w2"], self.y, self.topk_idx,
                    self.topk_gate, self.counts, self.ws, w_noise=w.get("w_noise"), noise=noise,
                    logit_bias=w.get("logit_bias"), importance=self.importance, load=self.load,
                    near_tie=self.near_tie, stream=stream)
        return self.y


__all__ = ["ACT", "DEVERR", "DTYPE", "GATING", "MoEConfig", "MoEError", "MoELayer", "STATUS", "lib",
           "make_config", "moe_capacity", "moe_combine", "moe_expert_ffn", "moe_forward",
           "moe_forward_workspace_size", "moe_get_error", "moe_permute", "moe_route",
           "moe_workspace_size", "workspace", "last_launch_count", "moe_bf16_to_f16",
           "moe_expert_ffn_grouped",
           "prepare_weights", "moe_permute_noalloc", "moe_expert_ffn_combine", "fused_combine",
           "moe_expert_ffn_gather", "moe_expert_ffn_combine_gather", "train_state",
           "backward_workspace", "moe_forward_train", "moe_backward"]
