"""Parity of the CUDA backward pass with the fp64 reference gradients.

moe_forward_train + moe_backward on seeded bf16 workloads against oracle/moe_backward.py
(whose gradients are pinned to central finite differences of the forward oracle's loss).
The reference recomputes the forward itself, so each case is chosen without near ties
(every token's k-th vs (k+1)-th score gap above 1e-4, checked here): both sides then route
every token alike.  Each gradient must be within max|err| / RMS <= 2e-2 of the reference
(the weight gradients expert by expert), the layer-output tolerance of the bf16 path: the expert products take bf16 operands (the
upstream gradient of each expert row and the hidden activations are rounded to 16 bits)
with fp32 accumulation; the router's gradients are fp32."""
import numpy as np
import pytest
import torch

import sparsely_gated_mixture_moe_b200 as moe
import workloads
from oracle import moe_backward as bwd
from oracle import moe_oracle as orc
from tests import gpu_harness as H
from workloads import Workload

pytestmark = pytest.mark.gpu

TOL = 2e-2

CASES = {
    # (workload, w_importance, w_load)
    "softmax_relu": (Workload("br", T=512, d_model=128, d_ff=256, E=8, k=2, act="relu",
                                      seed=1), 0.0, 0.0),
    "importance_gelu": (Workload("bi", T=700, d_model=128, d_ff=192, E=8, k=2, act="gelu",
                                         seed=1), 0.5, 0.0),
    "switch_capacity_f16": (Workload("bs", T=1024, d_model=128, d_ff=256, E=8, k=1, renorm=False,
                                     capacity_factor=1.0, act="gelu", hidden_f16=True), 0.0, 0.0),
    "noisy_losses": (Workload("bn", T=600, d_model=128, d_ff=128, E=16, k=2, gating="noisy_topk",
                              act="relu"), 0.3, 0.7),
    "zipf_bias_multitile": (workloads.WORKLOADS["zipf"].scaled(T=1536, d_model=256, d_ff=512,
                                                               seed=1), 0.0, 0.0),
    "k4_E32_capacity": (Workload("bk", T=800, d_model=64, d_ff=128, E=32, k=4, act="gelu",
                                 capacity_factor=0.8, seed=1), 0.2, 0.0),
}


def _dy(w):
    g = torch.Generator().manual_seed(77)
    return torch.randn(w.T, w.d_model, generator=g, dtype=torch.float32)


def _gpu_backward(w, inp, dy, w_imp, w_load):
    cfg = H.config_of(w)
    dev = moe.prepare_weights(cfg, H.to_device(inp))
    T, k, E, d, f = w.T, w.k, w.E, w.d_model, w.d_ff
    cu = "cuda"
    noisy = w.gating == "noisy_topk"
    o = {"y": torch.empty(T, d, device=cu), "idx": torch.empty(T, k, dtype=torch.int32, device=cu),
         "gate": torch.empty(T, k, device=cu), "counts": torch.empty(E, dtype=torch.int32, device=cu),
         "imp": torch.empty(E, device=cu), "load": torch.empty(E, device=cu) if noisy else None}
    state = moe.train_state(cfg)
    ws = moe.backward_workspace(cfg)
    moe.moe_forward_train(cfg, dev["x"], dev["w_gate"], dev["w1"], dev["w2"], o["y"], o["idx"],
                          o["gate"], o["counts"], state, ws, w_noise=dev.get("w_noise"),
                          noise=dev.get("noise"), logit_bias=dev.get("logit_bias"),
                          importance=o["imp"], load=o["load"])
    g = {"dx": torch.full((T, d), float("nan"), device=cu),
         "dw_gate": torch.full((E, d), float("nan"), device=cu),
         "dw_noise": torch.full((E, d), float("nan"), device=cu) if noisy else None,
         "dbias": torch.full((E,), float("nan"), device=cu) if "logit_bias" in dev else None,
         "dw1": torch.full((E, f, d), float("nan"), device=cu),
         "dw2": torch.full((E, d, f), float("nan"), device=cu),
         "dgates": torch.full((T, k), float("nan"), device=cu),
         "losses": torch.full((2,), float("nan"), device=cu)}
    moe.moe_backward(cfg, dev["x"], dev["w_gate"], dev["w1"], dev["w2"], o["idx"], o["gate"], state,
                     dy.cuda(), g["dx"], g["dw_gate"], g["dw1"], g["dw2"], g["dgates"], ws,
                     w_noise=dev.get("w_noise"), noise=dev.get("noise"),
                     logit_bias=dev.get("logit_bias"), importance=o["imp"], load=o["load"],
                     w_importance=w_imp, w_load=w_load, dw_noise=g["dw_noise"],
                     dlogit_bias=g["dbias"], losses=g["losses"])
    err = moe.moe_get_error(ws)
    out = {kk: (v.cpu() if v is not None else None) for kk, v in {**o, **g}.items()}
    out["device_error"] = err
    out["launches"] = moe.last_launch_count()
    # the training forward computes the same layer output as the inference forward
    layer = moe.MoELayer(cfg, {kk: v for kk, v in H.to_device(inp).items() if kk not in ("x", "noise")})
    y_inf = layer.forward(dev["x"], noise=dev.get("noise"))
    out["y_inference"] = y_inf.cpu()
    return out


@pytest.mark.parametrize("name", list(CASES))
def test_backward_matches_reference_gradients(name):
    w, w_imp, w_load = CASES[name]
    inp = workloads.make_inputs(w)
    r = orc.route(inp, w)
    assert np.all(r["gap"] > 1e-4), "case has near ties; choose another size"
    dy = _dy(w)
    g = _gpu_backward(w, inp, dy, w_imp, w_load)
    assert g["device_error"] == 0
    assert torch.equal(g["y"], g["y_inference"])
    assert np.array_equal(g["idx"].long().numpy(), r["idx"])
    ref = bwd.layer_backward(inp, w, dy.double().numpy(), w_importance=w_imp, w_load=w_load)
    rep = {}
    pairs = [("dx", "dx"), ("dw_gate", "dw_gate"), ("dw1", "dw1"), ("dw2", "dw2"),
             ("dgates", "dgates")]
    if w.gating == "noisy_topk":
        pairs.append(("dw_noise", "dw_noise"))
    if "logit_bias" in inp:
        pairs.append(("dbias", "dlogit_bias"))
    for got_key, ref_key in pairs:
        got, want = g[got_key].double().numpy(), ref[ref_key]
        if got_key in ("dw1", "dw2"):
            # each expert's weight gradient is its own parameter block: measured against
            # its own RMS (with Zipf-skewed expert sizes one global RMS is set by the many
            # small blocks and would stretch the hot expert's rounding error)
            e = max(H.rel_err(got[i], want[i]) for i in range(w.E) if np.any(want[i] != 0))
        else:
            e = H.rel_err(got, want)
        rep[got_key] = e
        assert e <= TOL, (got_key, e)
    # the auxiliary loss values
    if w_imp:
        imp = orc.importance(orc.dense_gates(w.T, w.E, r["idx"], r["gates"]))
        want = w_imp * bwd.cv_squared(imp)
        assert abs(float(g["losses"][0]) - want) <= 1e-4 * max(1.0, abs(want))
    if w_load:
        want = w_load * bwd.cv_squared(r["load"])
        assert abs(float(g["losses"][1]) - want) <= 1e-4 * max(1.0, abs(want))
    print(name, rep, "kernels", g["launches"])


def test_backward_rejects_unsupported():
    """fp32 layers and hierarchical gating have no backward here: refused up front."""
    c32 = moe.make_config(64, 64, 64, 4, 2, dtype="f32")
    assert moe.lib.moe_train_state_size(__import__("ctypes").byref(c32)) == 0
    ch = moe.make_config(64, 64, 64, 8, 2, gating="hierarchical", groups=2, k_primary=1)
    assert moe.lib.moe_backward_workspace_size(__import__("ctypes").byref(ch)) == 0
