"""Helpers of the GPU parity tests: run the library's steps on a workload and compare
each against the CPU oracle on the same inputs.

Step-wise parity feeds every oracle step the GPU's own upstream outputs (its expert
choices, its permuted rows), so a near tie in the router cannot cascade into later
steps; the end-to-end check follows the GPU's choice only at near ties (where the two
choices are both correct up to rounding) and the oracle's everywhere else.
"""
from __future__ import annotations

import numpy as np
import torch

import sparsely_gated_mixture_moe_b200 as moe
from oracle import moe_oracle as orc
import workloads

# max-abs error / RMS of the oracle output, by layer dtype (inputs and weights)
TOL = {"f32": 1e-5, "bf16": 2e-2}
BF16_U = 2.0 ** -8   # unit roundoff of bf16 (8 significant bits)
# absolute tolerance on fp32 gate values (fp32 softmax of fp32-accumulated scores)
GATE_ATOL = 2e-5
NEAR_TIE = 1e-4


def rel_err(got, want) -> float:
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    if want.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(want ** 2)))
    if rms == 0.0:
        return float(np.max(np.abs(got - want)))
    return float(np.max(np.abs(got - want))) / rms


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def config_of(w: workloads.Workload) -> moe.MoEConfig:
    return moe.make_config(w.T, w.d_model, w.d_ff, w.E, w.k, gating=w.gating, renorm=w.renorm,
                           capacity_factor=w.capacity_factor, act=w.act, dtype=w.dtype,
                           hidden_f16=w.hidden_f16, groups=w.groups, k_primary=w.k_primary)


def hidden_dtype(w):
    if w.dtype == "f32":
        return torch.float32
    return torch.float16 if w.hidden_f16 else torch.bfloat16


def to_device_prepared(w, inp, cfg=None):
    """Inputs on the GPU, weights as the forward pass takes them (fp16 w2 with fp16 h)."""
    return moe.prepare_weights(cfg or config_of(w), to_device(inp))


def to_device(inp):
    return {k: v.cuda() for k, v in inp.items()}


def run_steps(w, dev, cfg=None):
    """The four step calls on one stream; returns every output on the CPU."""
    cfg = cfg or config_of(w)
    dev = moe.prepare_weights(cfg, dev)
    T, k, E, d, f = w.T, w.k, w.E, w.d_model, w.d_ff
    dt = w.torch_dtype
    cu = "cuda"
    o = {
        "topk_idx": torch.full((T, k), -7, dtype=torch.int32, device=cu),
        "topk_gate": torch.full((T, k), float("nan"), dtype=torch.float32, device=cu),
        "near_tie": torch.full((T,), 9, dtype=torch.uint8, device=cu),
        "counts": torch.full((E,), -7, dtype=torch.int32, device=cu),
        "offsets": torch.full((E + 1,), -7, dtype=torch.int32, device=cu),
        "perm_src": torch.full((max(T * k, 1),), -7, dtype=torch.int32, device=cu),
        "slot_pos": torch.full((max(T * k, 1),), -7, dtype=torch.int32, device=cu),
        "x_perm": torch.zeros(max(T * k, 1), d, dtype=dt, device=cu),
        "h": torch.zeros(max(T * k, 1), f, dtype=hidden_dtype(w), device=cu),
        "y_perm": torch.zeros(max(T * k, 1), d, dtype=torch.float32, device=cu),
        "y": torch.full((T, d), float("nan"), dtype=torch.float32, device=cu),
    }
    noisy = w.gating == "noisy_topk"
    hier = w.gating == "hierarchical"
    o["importance"] = None if hier else torch.full((E,), float("nan"), device=cu)
    o["load"] = torch.full((E,), float("nan"), device=cu) if noisy and k < E else None
    ws = moe.workspace(cfg, cu)
    moe.moe_route(cfg, dev["x"], dev["w_gate"], o["topk_idx"], o["topk_gate"], ws,
                  w_noise=dev.get("w_noise"), noise=dev.get("noise"),
                  logit_bias=dev.get("logit_bias"), importance=o["importance"], load=o["load"],
                  near_tie=o["near_tie"])
    moe.moe_permute(cfg, o["topk_idx"], dev["x"], o["counts"], o["offsets"], o["perm_src"],
                    o["slot_pos"], o["x_perm"], ws)
    moe.moe_expert_ffn(cfg, o["x_perm"], o["offsets"], dev["w1"], dev["w2"], o["h"], o["y_perm"], ws)
    moe.moe_combine(cfg, o["y_perm"], o["slot_pos"], o["topk_gate"], o["y"], ws)
    if moe.fused_combine(cfg):
        # the fused FFN + combine step on the same permuted rows, into its own y
        o["y_fused"] = torch.full((T, d), float("nan"), dtype=torch.float32, device=cu)
        h2 = torch.zeros_like(o["h"])
        moe.moe_expert_ffn_combine(cfg, o["x_perm"], o["offsets"], o["perm_src"], o["slot_pos"],
                                   o["topk_gate"], dev["w1"], dev["w2"], h2, o["y_fused"], ws)
    # the same permutation with index arrays only, and the expert FFN gathering its rows
    # from x by perm_src (no x_perm): must give the same bits
    n = max(T * k, 1)
    gth = {"counts": torch.full((E,), -7, dtype=torch.int32, device=cu),
           "offsets": torch.full((E + 1,), -7, dtype=torch.int32, device=cu),
           "perm_src": torch.full((n,), -7, dtype=torch.int32, device=cu),
           "slot_pos": torch.full((n,), -7, dtype=torch.int32, device=cu),
           "h": torch.zeros(n, f, dtype=hidden_dtype(w), device=cu),
           "y_perm": torch.zeros(n, d, dtype=torch.float32, device=cu)}
    moe.moe_permute(cfg, o["topk_idx"], None, gth["counts"], gth["offsets"], gth["perm_src"],
                    gth["slot_pos"], None, ws)
    moe.moe_expert_ffn_gather(cfg, dev["x"], gth["perm_src"], gth["offsets"], dev["w1"], dev["w2"],
                              gth["h"], gth["y_perm"], ws)
    if moe.fused_combine(cfg):
        gth["y_fused"] = torch.full((T, d), float("nan"), dtype=torch.float32, device=cu)
        h3 = torch.zeros_like(o["h"])
        moe.moe_expert_ffn_combine_gather(cfg, dev["x"], gth["offsets"], gth["perm_src"],
                                          gth["slot_pos"], o["topk_gate"], dev["w1"], dev["w2"], h3,
                                          gth["y_fused"], ws)
    err = moe.moe_get_error(ws)
    out = {kk: (v.cpu() if v is not None else None) for kk, v in o.items()}
    out["gather"] = {kk: v.cpu() for kk, v in gth.items()}
    out["device_error"] = err
    return out


def check_gather_path(w, g, report):
    """The index-only permutation and the FFN that gathers its rows from x equal the
    x_perm path bit for bit (the same rows reach the same tensor-core tiles)."""
    gp = g["gather"]
    n = int(g["offsets"][-1]) if w.T else 0
    for key in ("counts", "offsets"):
        assert torch.equal(gp[key], g[key]), key
    assert torch.equal(gp["slot_pos"][: w.T * w.k], g["slot_pos"][: w.T * w.k])
    assert torch.equal(gp["perm_src"][:n], g["perm_src"][:n])
    assert torch.equal(gp["h"][:n], g["h"][:n]), "h differs between the gather and x_perm paths"
    assert torch.equal(gp["y_perm"][:n], g["y_perm"][:n]), "y_perm differs"
    if "y_fused" in gp:
        assert torch.equal(gp["y_fused"], g["y_fused"]), "fused y differs"
    report["gather_path"] = "equal"


def run_forward(w, dev, cfg=None):
    cfg = cfg or config_of(w)
    layer = moe.MoELayer(cfg, {kk: v for kk, v in dev.items() if kk not in ("x", "noise")})
    y = layer.forward(dev["x"], noise=dev.get("noise"))
    err = moe.moe_get_error(layer.ws)
    return {"y": y.cpu(), "topk_idx": layer.topk_idx.cpu(), "topk_gate": layer.topk_gate.cpu(),
            "counts": layer.counts.cpu(), "device_error": err,
            "importance": None if layer.importance is None else layer.importance.cpu(),
            "load": None if layer.load is None else layer.load.cpu()}


def reconcile_choice(w, r, idx_gpu):
    """The oracle's expert choice, except at near ties where the GPU's choice is taken
    after checking it is a correct one (its scores within the near-tie margin of the
    oracle's k-th score).  Returns (idx, n_near_tie, n_differ)."""
    idx_o = r["idx"]
    near = r["gap"] <= NEAR_TIE
    differ = ~np.all(idx_gpu == idx_o, axis=1)
    bad = differ & ~near
    assert not bad.any(), "expert choice differs on %d non-near-tie tokens, e.g. %s" % (
        int(bad.sum()), np.nonzero(bad)[0][:5])
    idx = idx_o.copy()
    if differ.any():
        s = -np.sort(-r["scores"], axis=1)
        kth = s[:, w.k - 1]
        rows = np.nonzero(differ)[0]
        chosen = np.take_along_axis(r["scores"][rows], idx_gpu[rows], axis=1)
        assert np.all(chosen >= kth[rows, None] - NEAR_TIE)
        assert all(len(set(v)) == w.k for v in idx_gpu[rows].tolist())
        idx[rows] = idx_gpu[rows]
    return idx, int(near.sum()), int(differ.sum())


def hier_gates_for(w, scores, idx):
    """The oracle's two-level gates for a given hierarchical choice idx [T, k] (e.g. the
    GPU's at a near tie): orc.gate_values at the primary level over the chosen groups,
    then within each chosen group over its chosen experts, multiplied."""
    a, k1 = w.groups, w.k_primary
    k2 = w.k // k1
    b = w.E // a
    T = idx.shape[0]
    prim = scores[:, :a]
    groups = idx[:, ::k2] // b                       # [T, k1]
    gp = orc.gate_values(prim, groups, True)
    out = np.zeros((T, w.k))
    rows = np.arange(T)
    for q in range(k1):
        g_ = groups[:, q]
        sec = np.stack([scores[t, a + g_[t] * b:a + (g_[t] + 1) * b] for t in range(T)])
        j = idx[:, q * k2:(q + 1) * k2] - g_[:, None] * b
        out[:, q * k2:(q + 1) * k2] = gp[:, q:q + 1] * orc.gate_values(sec, j, True)
    return out


def check_route_hier(w, inp, g, report):
    """Hierarchical gating: the GPU's choice equals the oracle's on every token whose gap
    at both levels exceeds the near-tie margin; elsewhere it must be a valid two-level
    choice (whole groups of k / k_primary distinct experts, distinct groups), which the
    later steps then follow.  Gates within GATE_ATOL of the oracle's for the choice."""
    r = orc.route(inp, w)
    idx_g = g["topk_idx"].long().numpy()
    assert idx_g.min() >= 0 and idx_g.max() < w.E
    near = r["gap"] <= NEAR_TIE
    differ = ~np.all(idx_g == r["idx"], axis=1)
    bad = differ & ~near
    assert not bad.any(), "expert choice differs on %d non-near-tie tokens, e.g. %s" % (
        int(bad.sum()), np.nonzero(bad)[0][:5])
    k2 = w.k // w.k_primary
    b = w.E // w.groups
    grp = idx_g // b
    for q in range(w.k_primary):   # each chosen group's block lies in one group
        blk = grp[:, q * k2:(q + 1) * k2]
        assert np.all(blk == blk[:, :1])
    assert all(len(set(v)) == w.k_primary for v in grp[:, ::k2].tolist())
    assert all(len(set(v)) == w.k for v in idx_g.tolist())
    idx = r["idx"].copy()
    idx[differ] = idx_g[differ]
    gates_o = hier_gates_for(w, r["scores"], idx)
    gerr = float(np.max(np.abs(g["topk_gate"].double().numpy() - gates_o))) if w.T else 0.0
    assert gerr <= GATE_ATOL, gerr
    nt = g["near_tie"].numpy().astype(bool)
    assert not np.any(nt & (r["gap"] > 2 * NEAR_TIE))
    assert not np.any(~nt & (r["gap"] < 0.5 * NEAR_TIE))
    report.update(near_ties=int(near.sum()), choice_differs=int(differ.sum()), gate_abs_err=gerr)
    return idx, gates_o


def check_route(w, inp, g, report):
    if w.gating == "hierarchical":
        return check_route_hier(w, inp, g, report)
    r = orc.route(inp, w)
    idx_g = g["topk_idx"].long().numpy()
    assert idx_g.min() >= 0 and idx_g.max() < w.E
    idx, n_near, n_diff = reconcile_choice(w, r, idx_g)
    renorm = True if w.gating == "noisy_topk" else w.renorm
    gates_o = orc.gate_values(r["scores"], idx, renorm)
    gerr = float(np.max(np.abs(g["topk_gate"].double().numpy() - gates_o))) if w.T else 0.0
    assert gerr <= GATE_ATOL, gerr
    nt = g["near_tie"].numpy().astype(bool)
    # the GPU's near-tie flag agrees with the oracle's gap away from the threshold
    assert not np.any(nt & (r["gap"] > 2 * NEAR_TIE))
    assert not np.any(~nt & (r["gap"] < 0.5 * NEAR_TIE))
    report.update(near_ties=n_near, choice_differs=n_diff, gate_abs_err=gerr)
    if g.get("importance") is not None:
        G = orc.dense_gates(w.T, w.E, idx, gates_o)
        imp = orc.importance(G)
        ierr = rel_err(g["importance"].double().numpy(), imp)
        assert ierr <= 1e-4, ierr
        report["importance_err"] = ierr
    if g.get("load") is not None:
        lerr = rel_err(g["load"].double().numpy(), r["load"])
        assert lerr <= 1e-4, lerr
        report["load_err"] = lerr
    return idx, gates_o


def check_permute(w, inp, g, report):
    idx_g = g["topk_idx"].long().numpy()
    C = orc.capacity(w.capacity_factor, w.T, w.k, w.E)
    counts, offsets, perm_src, slot_pos = orc.dispatch(idx_g, w.E, C)
    n = int(offsets[-1])
    assert g["counts"].tolist() == counts.tolist()
    assert g["offsets"].tolist() == offsets.tolist()
    assert g["slot_pos"][: w.T * w.k].tolist() == slot_pos.tolist()
    assert g["perm_src"][:n].tolist() == perm_src.tolist()
    # x_perm rows are byte copies of the token rows
    assert torch.equal(g["x_perm"][:n], inp["x"][torch.from_numpy(perm_src // w.k)])
    report.update(kept=n, dropped=w.T * w.k - n, capacity=C)
    return n


def gpu_hidden(w, g, rows):
    return f64(g["h"][rows])


def check_ffn(w, inp, g, n, report, rows=None):
    """y_perm and h of the GPU against the oracle's experts on the GPU's own x_perm.

    h is an intermediate stored in bf16 (or fp16): each element must be the
    oracle's value up to that storage's rounding, |dh| <= u |h| + 1e-4 rms(h), with
    u = 2^-8 for bf16 and 2^-11 for fp16 (fp32 path: 1e-5 of rms)."""
    off = g["offsets"].numpy()
    if rows is None:
        rows = list(range(n))
        h_o, y_o = orc.expert_ffn(f64(g["x_perm"][:n]), off, inp["w1"], inp["w2"], w.act)
    else:
        # the sampled rows, evaluated one expert at a time (each expert's weights are
        # converted to fp64 once)
        rows = sorted(rows)
        e_of = np.searchsorted(off, rows, side="right") - 1
        h_o = np.zeros((len(rows), w.d_ff))
        y_o = np.zeros((len(rows), w.d_model))
        for e in np.unique(e_of):
            sel = np.nonzero(e_of == e)[0]
            src = [rows[i] for i in sel]
            h1, y1 = orc.expert(f64(g["x_perm"][src]), inp["w1"][e], inp["w2"][e], w.act)
            h_o[sel] = h1
            y_o[sel] = y1
    h_g = gpu_hidden(w, g, rows)
    rms_h = float(np.sqrt(np.mean(h_o ** 2))) if h_o.size else 0.0
    if w.dtype == "bf16":
        u = 2.0 ** -11 if w.hidden_f16 else BF16_U
        bound = u * np.abs(h_o) + 1e-4 * rms_h
    else:
        bound = 1e-5 * rms_h + 1e-6 * np.abs(h_o)
    excess = float(np.max(np.abs(h_g - h_o) - bound)) if h_o.size else -1.0
    assert excess <= 0.0, excess
    eh = rel_err(h_g, h_o)
    ey = rel_err(f64(g["y_perm"][rows]), y_o)
    assert ey <= TOL[w.dtype], ey
    report.update(h_err=eh, y_perm_err=ey)


def check_combine(w, g, report, rows=None):
    sp = g["slot_pos"][: w.T * w.k].numpy()
    gates = g["topk_gate"].double().numpy()
    if rows is None:
        y_o = orc.combine(f64(g["y_perm"]), sp, gates, w.T, w.k)
        e = rel_err(f64(g["y"]), y_o)
    else:
        sub_sp = sp.reshape(w.T, w.k)[rows]
        yp = f64(g["y_perm"])
        y_o = np.zeros((len(rows), w.d_model))
        for n_, (t, s_row) in enumerate(zip(rows, sub_sp)):
            for j, s in enumerate(s_row):
                if s >= 0:
                    y_o[n_] += gates[t, j] * yp[s]
        e = rel_err(f64(g["y"][rows]), y_o)
    # fp32 in, fp32 accumulation, fp32 out on both paths
    assert e <= TOL["f32"], e
    report["combine_err"] = e
    if "y_fused" in g:
        if w.k == 1:
            # one fp32 product g * row on both paths: equal value for value
            assert torch.equal(g["y_fused"], g["y"]), float((g["y_fused"] - g["y"]).abs().max())
            report["fused_combine"] = "equal"
        else:
            # k = 2: the fused path adds the two rounded products (in-memory adds, which
            # commute); moe_combine folds the second product into its add (one FMA), so the
            # two differ by at most the rounding of that product
            yf, yc = g["y_fused"].double(), g["y"].double()
            assert torch.isfinite(yf).all()
            T_, k_ = w.T, w.k
            sp = g["slot_pos"].long().view(T_, k_)
            kept = (sp >= 0).double().unsqueeze(-1)
            yp = g["y_perm"].double()[sp.clamp(min=0)]                     # [T, k, d]
            mag = (g["topk_gate"].double().abs().view(T_, k_, 1) * yp.abs() * kept).sum(1)
            bound = 2.0 ** -22 * mag            # two roundings of size <= 2^-24 |term| each
            assert bool(((yf - yc).abs() <= bound).all()), float((yf - yc).abs().max())
            report["fused_combine"] = "within one rounding"


def oracle_layer_rows(w, inp, idx, gates, rows):
    """The oracle's layer output at the token rows ``rows`` for the expert choice ``idx``
    and gates ``gates``: capacity dispatch over all T tokens (orc.dispatch), then each
    kept assignment of a requested token through its expert (orc.expert, one call per
    expert over all its requested tokens), weighted by its gate and summed over j as in
    orc.combine.  The same arithmetic as orc.moe_forward_rows, batched by expert."""
    T, k = idx.shape
    C = orc.capacity(w.capacity_factor, T, w.k, w.E)
    counts, offsets, perm_src, slot_pos = orc.dispatch(idx, w.E, C)
    sp = slot_pos.reshape(T, k)
    rows = list(rows)
    pos = {t: i for i, t in enumerate(rows)}
    contrib = np.zeros((k, len(rows), w.d_model))
    by_e = {}
    for t in rows:
        for j in range(k):
            if sp[t, j] >= 0:
                by_e.setdefault(int(idx[t, j]), []).append((t, j))
    for e, tj in by_e.items():
        ts = [t for t, _ in tj]
        _, ye = orc.expert(f64(inp["x"][ts]), inp["w1"][e], inp["w2"][e], w.act)
        for (t, j), yrow in zip(tj, ye):
            contrib[j, pos[t]] = gates[t, j] * yrow
    y = np.zeros((len(rows), w.d_model))
    for j in range(k):   # the slot order of orc.combine
        y += contrib[j]
    return y, {"slot_pos": slot_pos, "C": C}


def check_end_to_end(w, inp, g, idx, gates, report, rows=None):
    tol = TOL[w.dtype]
    if rows is None:
        rows = list(range(w.T))
    y_o, r = oracle_layer_rows(w, inp, idx, gates, rows)
    e = rel_err(f64(g["y"][rows]), y_o)
    assert e <= tol, e
    # fully dropped tokens output exactly zero
    sp = r["slot_pos"].reshape(w.T, w.k)
    dropped = [i for i, t in enumerate(rows) if np.all(sp[t] < 0)]
    if dropped:
        assert torch.all(g["y"][[rows[i] for i in dropped]] == 0)
    report.update(y_err=e, fully_dropped_checked=len(dropped), y_rows_checked=len(rows))
