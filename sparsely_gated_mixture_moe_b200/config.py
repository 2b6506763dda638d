"""The moe_config struct of include/moe.h as a ctypes Structure, plus its enums."""
from __future__ import annotations

import ctypes

STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_CUDA",
          4: "MOE_ERR_DEVICE"}
GATING = {"softmax_topk": 0, "noisy_topk": 1, "hierarchical": 2}
ACT = {"relu": 0, "gelu": 1}
DTYPE = {"f32": 0, "bf16": 1}
DEVERR = {"expert_index": 1, "offsets": 2, "slot": 4, "timeout": 8}


class MoEError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__("%s (%s)" % (msg, STATUS.get(status, status)))
        self.status = status


class MoEConfig(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int64),
        ("d_model", ctypes.c_int32),
        ("d_ff", ctypes.c_int32),
        ("E", ctypes.c_int32),
        ("k", ctypes.c_int32),
        ("gating", ctypes.c_int32),
        ("renorm", ctypes.c_int32),
        ("capacity_factor", ctypes.c_float),
        ("act", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("hidden_f16", ctypes.c_int32),
        ("groups", ctypes.c_int32),
        ("k_primary", ctypes.c_int32),
        ("y_bf16", ctypes.c_int32),
    ]


def make_config(T, d_model, d_ff, E, k, gating="softmax_topk", renorm=True,
                capacity_factor=None, act="relu", dtype="bf16", hidden_f16=False, groups=None,
                k_primary=1, y_bf16=False) -> MoEConfig:
    """Build a MoEConfig from plain values (capacity_factor None = no limit; groups and
    k_primary only for hierarchical gating; y_bf16: the layer output in bf16, bf16 layers
    only)."""
    return MoEConfig(T=T, d_model=d_model, d_ff=d_ff, E=E, k=k, gating=GATING[gating],
                     renorm=1 if renorm else 0,
                     capacity_factor=0.0 if capacity_factor is None else float(capacity_factor),
                     act=ACT[act], dtype=DTYPE[dtype], hidden_f16=1 if hidden_f16 else 0,
                     groups=0 if groups is None else int(groups),
                     k_primary=int(k_primary) if gating == "hierarchical" else 0,
                     y_bf16=1 if y_bf16 else 0)
