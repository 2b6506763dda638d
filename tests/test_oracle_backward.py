"""Pins of the fp64 reference gradients (oracle/moe_backward.py).

Every gradient is checked against central finite differences of the forward oracle's
loss, entry by entry, on tiny inputs whose top-k choices, capacity drops and ReLU signs
cannot change under the perturbation (the checks assert the margins).  CV^2 is checked
against the standard library's population variance.  CPU only."""
import statistics

import numpy as np
import pytest

from oracle import moe_backward as bwd
from oracle import moe_oracle as orc
from workloads import Workload

EPS = 1e-6
CASES = {
    "softmax_renorm_relu": (Workload("a", T=6, d_model=5, d_ff=7, E=4, k=2, act="relu"), 0.0, 0.0, False),
    "softmax_importance": (Workload("b", T=7, d_model=4, d_ff=5, E=4, k=2, act="gelu"), 0.5, 0.0, False),
    "switch_top1_capacity": (Workload("c", T=8, d_model=4, d_ff=6, E=4, k=1, renorm=False,
                                      capacity_factor=1.0, act="gelu"), 0.0, 0.0, False),
    "bias_renorm": (Workload("d", T=6, d_model=4, d_ff=5, E=3, k=2, act="gelu"), 0.0, 0.0, True),
    "noisy_losses": (Workload("e", T=6, d_model=4, d_ff=6, E=5, k=2, gating="noisy_topk",
                              act="relu"), 0.3, 0.7, False),
}


def _inputs(w, seed, bias):
    rng = np.random.default_rng(seed)
    inp = {"x": rng.standard_normal((w.T, w.d_model)),
           "w_gate": rng.standard_normal((w.E, w.d_model)),
           "w1": rng.standard_normal((w.E, w.d_ff, w.d_model)) / np.sqrt(w.d_model),
           "w2": rng.standard_normal((w.E, w.d_model, w.d_ff)) / np.sqrt(w.d_ff)}
    if w.gating == "noisy_topk":
        inp["w_noise"] = rng.standard_normal((w.E, w.d_model)) * 0.5
        inp["noise"] = rng.standard_normal((w.T, w.E))
    if bias:
        inp["logit_bias"] = rng.standard_normal(w.E)
    return inp, rng.standard_normal((w.T, w.d_model))


def _loss(inp, w, dy, w_imp, w_load):
    r = orc.moe_forward(inp, w)
    L = float(np.sum(dy * r["y"]))
    if w_imp:
        G = orc.dense_gates(w.T, w.E, r["idx"], r["gates"])
        L += w_imp * bwd.cv_squared(orc.importance(G))
    if w_load:
        L += w_load * bwd.cv_squared(r["load"])
    return L


def _margins_ok(inp, w):
    """Top-k and every sorted neighbour of the scores well apart, ReLU inputs away from 0."""
    r = orc.moe_forward(inp, w)
    s = -np.sort(-r["scores"], axis=1)
    if np.min(s[:, :-1] - s[:, 1:]) < 1e-3:
        return False
    if w.act == "relu" and r["x_perm"].shape[0]:
        u = np.concatenate([r["x_perm"][a:b] @ inp["w1"][e].T
                            for e, (a, b) in enumerate(zip(r["offsets"][:-1], r["offsets"][1:]))
                            if b > a])
        if np.min(np.abs(u)) < 1e-3:
            return False
    return True


@pytest.mark.parametrize("name", list(CASES))
def test_gradients_match_finite_differences(name):
    w, w_imp, w_load, bias = CASES[name]
    for seed in range(50):
        inp, dy = _inputs(w, seed, bias)
        if _margins_ok(inp, w):
            break
    else:
        pytest.fail("no seed with clear margins")
    g = bwd.layer_backward(inp, w, dy, w_importance=w_imp, w_load=w_load)
    assert abs(g["loss"] - _loss(inp, w, dy, w_imp, w_load)) <= 1e-12 * max(1.0, abs(g["loss"]))
    params = {"x": "dx", "w_gate": "dw_gate", "w1": "dw1", "w2": "dw2"}
    if bias:
        params["logit_bias"] = "dlogit_bias"
    if w.gating == "noisy_topk":
        params["w_noise"] = "dw_noise"
    for pname, gname in params.items():
        an = g[gname]
        assert an is not None and an.shape == np.shape(inp[pname])
        fd = np.zeros_like(an)
        base = inp[pname]
        for i in np.ndindex(an.shape):
            for sgn in (1.0, -1.0):
                pert = base.copy()
                pert[i] += sgn * EPS
                inp[pname] = pert
                fd[i] += sgn * _loss(inp, w, dy, w_imp, w_load)
            inp[pname] = base
        fd /= 2.0 * EPS
        scale = max(1.0, float(np.max(np.abs(fd))))
        err = float(np.max(np.abs(fd - an))) / scale
        assert err <= 1e-6, (name, pname, err)


def test_cv_squared_is_population_variance_over_squared_mean():
    v = np.array([3.0, 1.0, 4.0, 1.0, 5.0, 9.0])
    assert bwd.cv_squared(v) == pytest.approx(statistics.pvariance(v) / statistics.mean(v) ** 2,
                                              rel=1e-14)
    # and its gradient against central differences
    gr = bwd.cv_squared_grad(v)
    for i in range(v.size):
        e = np.zeros_like(v)
        e[i] = EPS
        fd = (bwd.cv_squared(v + e) - bwd.cv_squared(v - e)) / (2 * EPS)
        assert gr[i] == pytest.approx(fd, abs=1e-8)


def test_uniform_importance_has_zero_cv_and_zero_gradient():
    v = np.full(5, 2.5)
    assert bwd.cv_squared(v) == 0.0
    assert np.all(bwd.cv_squared_grad(v) == 0.0)
