"""Seeded synthetic inputs for the sparsely-gated Mixture-of-Experts layer forward.

This module is shared by the CUDA path's tests and benchmark and by the CPU oracle's
tests. It holds shapes, seeds and value distributions only: it performs none of the
layer's arithmetic (no router product, gating, dispatch, expert FFN or combine).

Every tensor is drawn from its own ``torch.Generator('cpu')`` seeded with
``seed * 100 + tensor_id``, sampled in fp32 and then rounded (round-to-nearest-even)
to the storage dtype, so the inputs are bit-identical on every machine.

Distributions (fan_in is the contraction length of the product the tensor enters):
  x ~ N(0, 1)                        [T, d_model]
  w_gate, w_noise ~ N(0, 1/d_model)  [E, d_model]  (the gating matrices W_g, W_noise of
                                       "Noisy Top-K Gating", stored transposed: one row
                                       per expert, so each row is contiguous along d_model;
                                       [groups + E, d_model] for hierarchical gating)
  w1 ~ N(0, 1/d_model)               [E, d_ff, d_model]   up-projection, K-major
  w2 ~ N(0, 1/d_ff)                  [E, d_model, d_ff]   down-projection, K-major
  noise ~ N(0, 1) fp32               [T, E]  the StandardNormal() draws of noisy gating,
                                       supplied as an input so both sides use the same draws
  logit_bias fp32                    [E]  only for the skewed workload: b_e = beta*ln(p_e),
                                       p_e proportional to (e+1)^-s (Zipf).  beta is a stored
                                       constant (zipf_beta.json) written by
                                       oracle/calibrate_zipf.py.
"""
from __future__ import annotations

import dataclasses
import json
import math
import os
from typing import Dict, Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))

# tensor ids: each tensor gets its own stream so adding one never shifts another
TENSOR_IDS = {"x": 1, "w_gate": 2, "w_noise": 3, "w1": 4, "w2": 5, "noise": 6}


@dataclasses.dataclass(frozen=True)
class Workload:
    """One layer-forward problem: shapes, gating rule, capacity and dtype.

    gating: "softmax_topk" (softmax over experts, keep top k) or "noisy_topk"
            (Shazeer et al. noisy top-k gating).
    renorm: for softmax_topk, True = gates are Softmax(KeepTopK(logits, k)) (the
            renormalised top-k); False = each chosen expert's gate is its probability
            under the softmax over all experts (Switch top-1 rule).
    capacity_factor: None = no limit; else C = ceil(cf * T * k / E) per expert.
    zipf_s: None, or the Zipf exponent of the per-expert logit bias.
    groups, k_primary: hierarchical gating ("hierarchical"): E experts in `groups` groups
            of E / groups; the primary gate keeps k_primary groups and each chosen group's
            gate keeps k / k_primary of its experts.  w_gate then has groups + E rows: the
            primary gating rows, then each group's secondary gating rows.
    hidden_f16: store the expert hidden activations in fp16 (11 significant bits)
            instead of bf16 (8), with W2 re-encoded to fp16 for the second product.  The
            Switch workload needs it to keep the layer output within max|err|/RMS <= 2e-2:
            its top-1 gates vary several-fold between tokens, which stretches the
            max-to-RMS ratio of the error that a bf16 rounding of h leaves.
    """

    name: str
    T: int
    d_model: int
    d_ff: int
    E: int
    k: int
    gating: str = "softmax_topk"
    renorm: bool = True
    capacity_factor: Optional[float] = None
    act: str = "relu"
    dtype: str = "bf16"
    zipf_s: Optional[float] = None
    hidden_f16: bool = False
    groups: Optional[int] = None
    k_primary: int = 1
    seed: int = 0

    def scaled(self, **kw) -> "Workload":
        """Same workload with some fields replaced (used for small parity cases)."""
        return dataclasses.replace(self, **kw)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def describe(self) -> dict:
        return dataclasses.asdict(self)


# The five problems: a tiny fp32 check, Switch top-1 with capacity, Shazeer noisy top-4,
# GShard top-2 with capacity, and a skewed dropless top-2 stress case.
WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", T=512, d_model=64, d_ff=256, E=8, k=2, gating="softmax_topk",
                     renorm=True, capacity_factor=None, act="relu", dtype="f32"),
    "switch": Workload("switch", T=16384, d_model=768, d_ff=3072, E=128, k=1,
                       gating="softmax_topk", renorm=False, capacity_factor=1.25,
                       act="gelu", dtype="bf16", hidden_f16=True),
    "noisy": Workload("noisy", T=8192, d_model=512, d_ff=1024, E=256, k=4,
                      gating="noisy_topk", renorm=True, capacity_factor=None,
                      act="relu", dtype="bf16"),
    "gshard": Workload("gshard", T=32768, d_model=1024, d_ff=8192, E=64, k=2,
                       gating="softmax_topk", renorm=True, capacity_factor=2.0,
                       act="gelu", dtype="bf16"),
    "zipf": Workload("zipf", T=65536, d_model=1024, d_ff=4096, E=16, k=2,
                     gating="softmax_topk", renorm=True, capacity_factor=None,
                     act="gelu", dtype="bf16", zipf_s=1.2),
    # a two-level (hierarchical) layer at the noisy workload's size: 8 groups of 16
    # experts, 2 groups and 2 experts in each kept ("MoE-H" keeps 2 per level)
    "hierarchical": Workload("hierarchical", T=8192, d_model=512, d_ff=1024, E=128, k=4,
                             gating="hierarchical", groups=8, k_primary=2, act="relu",
                             dtype="bf16"),
}
ORDER = ["tiny", "switch", "noisy", "gshard", "zipf", "hierarchical"]


def zipf_beta() -> float:
    """The stored bias scale beta for the skewed workload (see oracle/calibrate_zipf.py)."""
    with open(os.path.join(_HERE, "zipf_beta.json")) as f:
        return float(json.load(f)["beta"])


def zipf_probs(E: int, s: float) -> torch.Tensor:
    """Target Zipf expert shares p_e proportional to (e+1)^-s, fp64."""
    w = torch.tensor([(e + 1.0) ** (-s) for e in range(E)], dtype=torch.float64)
    return w / w.sum()


def _normal(shape, tensor: str, seed: int, std: float) -> torch.Tensor:
    g = torch.Generator("cpu")
    g.manual_seed(seed * 100 + TENSOR_IDS[tensor])
    out = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        out.mul_(std)
    return out


def make_inputs(w: Workload, beta: Optional[float] = None) -> Dict[str, torch.Tensor]:
    """Draw every input of workload ``w`` on the CPU, in its storage dtype.

    Returns x, w_gate, w1, w2 always; w_noise and noise for noisy gating; logit_bias
    for the Zipf-skewed workload (beta defaults to the stored calibration).
    """
    dt = w.torch_dtype
    d, f, E, T = w.d_model, w.d_ff, w.E, w.T
    out: Dict[str, torch.Tensor] = {}
    out["x"] = _normal((T, d), "x", w.seed, 1.0).to(dt)
    n_gate = E + (w.groups if w.gating == "hierarchical" else 0)
    out["w_gate"] = _normal((n_gate, d), "w_gate", w.seed, 1.0 / math.sqrt(d)).to(dt)
    if w.gating == "noisy_topk":
        out["w_noise"] = _normal((E, d), "w_noise", w.seed, 1.0 / math.sqrt(d)).to(dt)
        out["noise"] = _normal((T, E), "noise", w.seed, 1.0)
    out["w1"] = _normal((E, f, d), "w1", w.seed, 1.0 / math.sqrt(d)).to(dt)
    out["w2"] = _normal((E, d, f), "w2", w.seed, 1.0 / math.sqrt(f)).to(dt)
    if w.zipf_s is not None:
        b = zipf_beta() if beta is None else beta
        out["logit_bias"] = (b * torch.log(zipf_probs(E, w.zipf_s))).to(torch.float32)
    return out


def make_x(w: Workload) -> torch.Tensor:
    """Only the token activations of ``w`` (cheap when the weights are not needed)."""
    return _normal((w.T, w.d_model), "x", w.seed, 1.0).to(w.torch_dtype)
