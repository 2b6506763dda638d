"""Plain, slow fp64 CPU reference of the gradients of the sparsely-gated MoE layer.

TEST INFRASTRUCTURE, like moe_oracle: only the tests may import it; it shares no code
with the CUDA library.  It is the reference for the layer's backward pass, which the
CUDA library does not implement yet.  It recomputes the forward with moe_oracle's
functions and takes the steps back in reverse order.

Loss whose gradients are returned (dy is the gradient of the loss with respect to y):
    L = sum(dy * y) + w_importance * CV(Importance(X))^2 + w_load * CV(Load(X))^2
[SGMoE "Load-Balancing-Losses": the auxiliary losses are a scaling factor times the
squared coefficient of variation of Importance and of Load].

Readings where the pages are silent:
  * The top-k choice and the capacity drop are piecewise constant: no gradient flows
    through which experts are chosen or kept, only through the values.
  * The noise draws are inputs, not parameters.
  * CV is std / mean with the population standard deviation.
  * kth_excluding(H, k, i) is one entry of H (the k-th or (k+1)-th largest of the row);
    its gradient flows to that entry.
  * Importance sums the gates of every chosen expert before the capacity drop (as the
    forward oracle computes it).

parity pins: tests/test_oracle_backward.py checks every gradient against central finite
differences of moe_oracle's forward loss in fp64.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf

from oracle import moe_oracle as orc

_f64 = orc._f64


def cv_squared(v):
    """CV(v)^2 = var(v) / mean(v)^2 with the population variance."""
    v = _f64(v)
    m = float(np.mean(v))
    return float(np.var(v)) / (m * m)


def cv_squared_grad(v):
    """d CV(v)^2 / d v_i = 2 (v_i - m) / (n m^2) - 2 var / (n m^3)."""
    v = _f64(v)
    n = v.size
    m = float(np.mean(v))
    var = float(np.var(v))
    return 2.0 * (v - m) / (n * m * m) - 2.0 * var / (n * m ** 3)


def act_grad(u, act):
    """Derivative of the expert activation at the pre-activation u: ReLU' = [u > 0];
    GELU'(u) = Phi(u) + u * phi(u) for the exact erf form."""
    u = _f64(u)
    if act == "relu":
        return (u > 0.0).astype(np.float64)
    phi = np.exp(-0.5 * u * u) / math.sqrt(2.0 * math.pi)
    return 0.5 * (1.0 + erf(u / math.sqrt(2.0))) + u * phi


def softmax_backward(p, dp):
    """Rows of p = softmax(v): dv = p * (dp - <p, dp>)."""
    return p * (dp - np.sum(p * dp, axis=1, keepdims=True))


def sigmoid(z):
    """Softplus'(z)."""
    z = _f64(z)
    return 0.5 * (1.0 + np.tanh(0.5 * z))


def layer_backward(inp, w, dy, w_importance=0.0, w_load=0.0):
    """Gradients of L (above) with respect to x, w_gate, logit_bias, w_noise, w1 and w2.

    inp: the forward inputs (as for moe_oracle.moe_forward); w: the workload fields
    (gating, k, E, renorm, capacity_factor, act); dy [T, d].  Returns a dict with the
    loss and dx, dw_gate, dlogit_bias (None without a bias), dw_noise (None unless noisy),
    dw1, dw2, and the gate gradient dgates [T, k]."""
    x = _f64(inp["x"])
    wg = _f64(inp["w_gate"])
    w1, w2 = _f64(inp["w1"]), _f64(inp["w2"])
    bias = inp.get("logit_bias")
    dy = _f64(dy)
    T, d = x.shape
    E, k = w.E, w.k
    noisy = w.gating == "noisy_topk"
    rows = np.arange(T)[:, None]

    # ---- forward, keeping what the backward needs
    l = orc.router_logits(x, wg, bias)
    if noisy:
        wn, noise = _f64(inp["w_noise"]), _f64(inp["noise"])
        z = x @ wn.T
        s = orc.softplus(z)
        scores = l + noise * s
    else:
        scores = l
    idx = orc.top_k(scores, k)
    renorm = True if noisy else w.renorm
    p = orc.softmax(orc.keep_top_k(scores, idx)) if renorm else orc.softmax(scores)
    gates = p[rows, idx]
    C = orc.capacity(w.capacity_factor, T, k, E)
    _, offsets, perm_src, slot_pos = orc.dispatch(idx, E, C)
    x_perm = x[perm_src // k]
    n = x_perm.shape[0]
    u = np.zeros((n, w1.shape[1]))
    h = np.zeros_like(u)
    o = np.zeros((n, d))
    act = orc.ACTS[w.act]
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b > a:
            u[a:b] = x_perm[a:b] @ w1[e].T
            h[a:b] = act(u[a:b])
            o[a:b] = h[a:b] @ w2[e].T
    y = orc.combine(o, slot_pos, gates, T, k)
    loss = float(np.sum(dy * y))

    # ---- combine: y_t = sum_j G_tj o_slot(t,j)
    sp = np.asarray(slot_pos).reshape(T, k)
    d_o = np.zeros_like(o)
    dgates = np.zeros((T, k))
    for j in range(k):
        keep = sp[:, j] >= 0
        slots = sp[keep, j]
        d_o[slots] = gates[keep, j][:, None] * dy[keep]
        dgates[keep, j] = np.sum(dy[keep] * o[slots], axis=1)

    # ---- experts: o = act(x_perm W1_e^T) W2_e^T on each expert's kept rows
    dw1, dw2 = np.zeros_like(w1), np.zeros_like(w2)
    dx_perm = np.zeros_like(x_perm)
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b > a:
            dw2[e] = d_o[a:b].T @ h[a:b]
            du = (d_o[a:b] @ w2[e]) * act_grad(u[a:b], w.act)
            dw1[e] = du.T @ x_perm[a:b]
            dx_perm[a:b] = du @ w1[e]
    dx = np.zeros_like(x)
    np.add.at(dx, perm_src // k, dx_perm)

    # ---- auxiliary losses
    dgates_all = dgates.copy()
    if w_importance:
        imp = orc.importance(orc.dense_gates(T, E, idx, gates))
        loss += w_importance * cv_squared(imp)
        dimp = w_importance * cv_squared_grad(imp)
        dgates_all += dimp[idx]
    dl_load = np.zeros_like(scores)
    ds_load = np.zeros_like(scores)
    dH_load = np.zeros_like(scores)
    if w_load:
        if not noisy or k >= E:
            raise ValueError("the load loss needs noisy gating with k < E")
        kex = orc.kth_excluding(scores, k)
        zeta = (l - kex) / s
        P = orc.std_normal_cdf(zeta)
        ld = orc.load(P)
        loss += w_load * cv_squared(ld)
        dP = np.broadcast_to(w_load * cv_squared_grad(ld), P.shape)
        g = dP * np.exp(-0.5 * zeta * zeta) / math.sqrt(2.0 * math.pi)
        dl_load = g / s
        ds_load = -g * zeta / s
        # kth_excluding(H, k, i) is H at the (k+1)-th largest entry when H_i is among the
        # top k (H_i >= k-th largest value), else at the k-th largest
        order = np.argsort(-scores, axis=1, kind="stable")
        hk = np.take_along_axis(scores, order[:, k - 1:k], axis=1)
        src = np.where(scores >= hk, order[:, k:k + 1], order[:, k - 1:k])
        np.add.at(dH_load, (np.broadcast_to(rows, src.shape), src), -g / s)

    # ---- gates -> scores (softmax over the chosen experts, or over all for the Switch gate)
    dp = np.zeros_like(p)
    np.add.at(dp, (np.broadcast_to(rows, idx.shape), idx), dgates_all)
    dscores = softmax_backward(p, dp)

    # ---- scores -> router parameters and x
    if noisy:
        dH = dscores + dH_load
        dl = dH + dl_load
        dz = (dH * noise + ds_load) * sigmoid(z)
        dw_noise = dz.T @ x
        dx += dz @ wn
    else:
        dl = dscores
        dw_noise = None
    dw_gate = dl.T @ x
    dx += dl @ wg
    dbias = np.sum(dl, axis=0) if bias is not None else None
    return {"loss": loss, "dx": dx, "dw_gate": dw_gate, "dlogit_bias": dbias,
            "dw_noise": dw_noise, "dw1": dw1, "dw2": dw2, "dgates": dgates}
