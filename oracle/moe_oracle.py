"""Plain, slow fp64 CPU oracle of the sparsely-gated Mixture-of-Experts layer forward.

TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU-baseline
leg may import this module. It shares no code with the CUDA library and never imports
it; it reads inputs in their stored dtype upcast exactly to fp64.

Sources (pages by title, then section):
  [SGMoE]  "Outrageously Large Neural Networks: The Sparsely-Gated Mixture-of-Experts
           Layer" (summary page): "Methode (mit den Schlüsselgleichungen)" for the layer
           output y = sum_i G(x)_i E_i(x); "Noisy Top-K Gating" for H, KeepTopK and
           G = Softmax(KeepTopK(H, k)); "Load-Balancing-Losses" for Importance, P(x, i)
           with kth_excluding, and Load; "Schlüsselbegriffe" (experts are feed-forward
           sub-networks).
  [Switch] "Switch Transformer" page: the switch_routing pseudo-implementation (router
           logits, softmax over experts, keep the top-1 probability as the gate, dispatch
           by gather).
  [Setups] "moe paper models" page, Table 2 (TOP-K and capacity columns: capacity
           factors 1/1.5/2x, 1.25, 2).

Readings where the pages are silent or garbled:
  * KeepTopK keeps v_i when v_i is among the k largest entries and sets the rest to -inf.
  * Ties in the top-k choice go to the lowest expert index.
  * The top-k decision is taken on the scores rounded to fp32 (the kernel's precision);
    all values (gates, outputs) are then computed in fp64.  The k-th vs (k+1)-th gap is
    reported in fp64 so callers can exclude near ties.
  * Switch top-1 selects on the logits (softmax is monotone) and the gate is the chosen
    expert's probability under the softmax over all experts, not renormalised.
  * kth_excluding(H, k, i) is the k-th largest value of {H_j : j != i}.
  * Capacity C = ceil(cf * T * k / E) with cf taken as the fp32 value the config holds;
    per expert the C assignments of lowest flattened index t*k + j are kept; a dropped
    assignment contributes zero and gates are not renormalised after a drop.
  * Experts are E_i(x) = W2_i act(W1_i x) with no biases; GELU is the exact erf form.
  * Hierarchical MoE (one sentence on the page, "MoE-H" in the setups table): two levels
    of the page's top-k gate without noise, a primary gate over groups and a secondary
    gate over each chosen group's experts; an assignment's gate is the product of the
    two levels' gates, and the layer sums over both levels' chosen entries.

parity pins: every function below is pinned by tests/test_oracle_pins.py against hand
derivations, library routines (torch.nn.functional, scipy.stats) or brute force.
"""
from __future__ import annotations

from fractions import Fraction
import math
from typing import Dict, Optional

import numpy as np
from scipy.special import erf, erfc


def _f64(a):
    """fp64 numpy copy of a numpy array or a CPU torch tensor (bf16 upcasts exactly)."""
    if hasattr(a, "detach"):
        return a.detach().to("cpu").double().numpy()
    return np.asarray(a, np.float64)

# ----------------------------------------------------------------------------- gating


def router_logits(x, w_gate, logit_bias=None):
    """Clean gating logits x . W_g  [SGMoE "Noisy Top-K Gating"; Switch router logits].

    x [T, d]; w_gate [E, d] holds W_g transposed (one row per expert); logit_bias [E]
    or None (added to every token's logits).  Returns fp64 [T, E].
    """
    l = _f64(x) @ _f64(w_gate).T
    if logit_bias is not None:
        l = l + _f64(logit_bias)[None, :]
    return l


def softplus(z):
    """Softplus(z) = ln(1 + e^z), written in the overflow-free form max(z,0)+ln(1+e^-|z|)."""
    z = _f64(z)
    return np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z)))


def noisy_logits(x, w_gate, w_noise, noise, logit_bias=None):
    """H(x)_i = (x.W_g)_i + StandardNormal() * Softplus((x.W_noise)_i)  [SGMoE "Noisy Top-K
    Gating"].  The StandardNormal draws are the supplied ``noise`` [T, E].

    Returns (clean logits l, softplus term s, noisy logits H), all fp64 [T, E].
    """
    l = router_logits(x, w_gate, logit_bias)
    s = softplus(_f64(x) @ _f64(w_noise).T)
    H = l + _f64(noise) * s
    return l, s, H


def top_k(v, k):
    """Indices of the k largest entries of each row of v, largest first.

    The decision is taken on v rounded to fp32; ties go to the lowest index (a stable
    sort on the negated values keeps equal entries in ascending index order).
    """
    v32 = _f64(v).astype(np.float32)
    order = np.argsort(-v32, axis=1, kind="stable")
    return order[:, :k].astype(np.int64)


def topk_gap(v, k):
    """fp64 gap between the k-th and (k+1)-th largest entries of each row (inf if k == E).
    Rows whose gap is <= 1e-4 are near ties: two correct top-k choices may differ there."""
    v = _f64(v)
    if k >= v.shape[1]:
        return np.full(v.shape[0], np.inf)
    s = -np.sort(-v, axis=1)
    return s[:, k - 1] - s[:, k]


def keep_top_k(v, idx):
    """KeepTopK(v, k): v_i where i is one of the chosen top-k indices, -inf elsewhere
    [SGMoE "Noisy Top-K Gating"]."""
    v = _f64(v)
    out = np.full_like(v, -np.inf)
    rows = np.arange(v.shape[0])[:, None]
    out[rows, idx] = v[rows, idx]
    return out


def softmax(v):
    """Row softmax; entries at -inf get probability 0."""
    v = _f64(v)
    m = np.max(v, axis=1, keepdims=True)
    e = np.exp(v - m)
    return e / np.sum(e, axis=1, keepdims=True)


def gate_values(scores, idx, renorm):
    """Gate of each chosen expert.

    renorm=True : G(x) = Softmax(KeepTopK(scores, k)) evaluated at the chosen indices
                  [SGMoE "Noisy Top-K Gating"].
    renorm=False: the chosen expert's probability under the softmax over all experts
                  [Switch: softmax, then top-1 weight kept as the gate].
    ``idx`` may be any valid choice (e.g. another side's choice at a near tie).
    """
    rows = np.arange(idx.shape[0])[:, None]
    if renorm:
        G = softmax(keep_top_k(scores, idx))
    else:
        G = softmax(scores)
    return G[rows, idx]


def kth_excluding(H, k):
    """kth_excluding(H, k, i) for every token and every expert i: the k-th largest value of
    {H_j : j != i}  [SGMoE "Load-Balancing-Losses"].

    With h_(1) >= h_(2) >= ... the sorted row, removing H_i leaves the k-th largest at
    h_(k+1) when H_i >= h_(k) (H_i sits among the top k values) and at h_(k) otherwise.
    Requires k < E.  Returns fp64 [T, E].
    """
    H = _f64(H)
    T, E = H.shape
    if not 1 <= k < E:
        raise ValueError("kth_excluding needs 1 <= k < E")
    s = -np.sort(-H, axis=1)
    hk = s[:, k - 1:k]
    hk1 = s[:, k:k + 1]
    return np.where(H >= hk, hk1, hk)


def std_normal_cdf(z):
    """Phi(z) = erfc(-z / sqrt 2) / 2."""
    return 0.5 * erfc(-_f64(z) / math.sqrt(2.0))


def load_probability(l, s, H, k):
    """P(x, i) = Phi(((x.W_g)_i - kth_excluding(H(x), k, i)) / Softplus((x.W_noise)_i))
    [SGMoE "Load-Balancing-Losses"]: clean logits in the numerator, noisy H for
    kth_excluding, the softplus noise scale in the denominator.  fp64 [T, E]."""
    return std_normal_cdf((_f64(l) - kth_excluding(H, k)) / _f64(s))


def dense_gates(T, E, idx, gates, slot_pos=None):
    """G(x) as a dense [T, E] matrix: the gate at each chosen expert, 0 elsewhere; with
    slot_pos given, dropped assignments (slot_pos == -1) also get 0."""
    G = np.zeros((T, E))
    k = idx.shape[1]
    for j in range(k):
        g = gates[:, j].copy()
        if slot_pos is not None:
            g[slot_pos.reshape(T, k)[:, j] < 0] = 0.0
        G[np.arange(T), idx[:, j]] += g
    return G


def importance(G):
    """Importance(X) = sum over the batch of G(x)  [SGMoE "Load-Balancing-Losses"]. [E]"""
    return np.sum(_f64(G), axis=0)


def load(P):
    """Load(X)_i = sum over the batch of P(x, i)  [SGMoE "Load-Balancing-Losses"]. [E]"""
    return np.sum(_f64(P), axis=0)


# ------------------------------------------------------------ hierarchical gating


def hierarchical_gates(l, groups, k_primary, k_group):
    """Two-level gating of a hierarchical MoE [SGMoE "Schlüsselbegriffe": a primary gating
    network routes each input to secondary MoE groups; Setups Table 2: "MoE-H" with 4 or
    2 chosen per level].

    l [T, a + a*b] holds the clean logits of the primary gate over the a groups (columns
    0 .. a-1), then group i's secondary logits over its b experts (columns a + i*b ..
    a + i*b + b - 1).  Each level is the page's top-k gate without noise:
      G_p(x)   = Softmax(KeepTopK(primary logits, k_primary))        over the a groups
      G_i(x)   = Softmax(KeepTopK(group i's logits, k_group))        over its b experts
      y        = sum_i G_p(x)_i sum_j G_i(x)_j E_{i,j}(x)
    so a token has k_primary * k_group assignments; expert (i, j) has the flat index
    i*b + j and the gate G_p(x)_i * G_i(x)_j.  Chosen groups are listed by descending
    primary score, and within a group the chosen experts by descending secondary score
    (ties to the lowest index at both levels, decided on fp32 scores as top_k does).

    Returns (idx [T, k_primary*k_group] int64, gates [T, k_primary*k_group], gap [T]):
    gap is the smallest k-th vs (k+1)-th gap among the primary scores and the chosen
    groups' secondary scores (a near tie at either level where it is <= 1e-4)."""
    l = _f64(l)
    T = l.shape[0]
    a = int(groups)
    b = (l.shape[1] - a) // a
    if l.shape[1] != a + a * b or not (1 <= k_primary <= a and 1 <= k_group <= b):
        raise ValueError("bad hierarchical gating shape")
    prim = l[:, :a]
    sec = l[:, a:].reshape(T, a, b)
    chosen = top_k(prim, k_primary)                  # [T, k_primary]
    g_prim = gate_values(prim, chosen, True)         # G_p at the chosen groups
    gap = topk_gap(prim, k_primary)
    k = k_primary * k_group
    idx = np.zeros((T, k), np.int64)
    gates = np.zeros((T, k))
    rows = np.arange(T)
    for q in range(k_primary):
        g = chosen[:, q]
        s = sec[rows, g, :]                          # [T, b]: the chosen group's logits
        j = top_k(s, k_group)
        idx[:, q * k_group:(q + 1) * k_group] = g[:, None] * b + j
        gates[:, q * k_group:(q + 1) * k_group] = g_prim[:, q:q + 1] * gate_values(s, j, True)
        gap = np.minimum(gap, topk_gap(s, k_group))
    return idx, gates, gap


def hierarchical_dense_gates(l, groups, k_primary, k_group):
    """G(x) of the hierarchical layer as a dense [T, a*b] matrix, by its definition: the
    dense primary gate Softmax(KeepTopK(., k_primary)) over the groups times each
    group's dense secondary gate Softmax(KeepTopK(., k_group)), evaluated for every group
    (unchosen groups get primary weight 0)."""
    l = _f64(l)
    T = l.shape[0]
    a = int(groups)
    b = (l.shape[1] - a) // a
    prim = l[:, :a]
    Gp = softmax(keep_top_k(prim, top_k(prim, k_primary)))       # [T, a]
    G = np.zeros((T, a * b))
    for i in range(a):
        s = l[:, a + i * b:a + (i + 1) * b]
        Gi = softmax(keep_top_k(s, top_k(s, k_group)))            # [T, b]
        G[:, i * b:(i + 1) * b] = Gp[:, i:i + 1] * Gi
    return G


# ------------------------------------------------------------------ capacity, dispatch


def capacity(cf, T, k, E):
    """Per-expert capacity C = ceil(cf * T * k / E) in exact rational arithmetic on the
    fp32 value of cf; None when cf is None or <= 0 (no limit).  [Setups, Table 2:
    capacity factors; the formula is the plainest reading of "capacity factor".]"""
    if cf is None or cf <= 0:
        return None
    q = Fraction(float(np.float32(cf))) * T * k / E
    return int(math.ceil(q))


def dispatch(idx, E, C=None):
    """Stable counting sort of the T*k assignments by expert, with capacity truncation.

    Assignment a = t*k + j goes to expert idx[t, j].  Within an expert, assignments keep
    ascending a (token order) and only the first C are kept [Switch: dispatch is a
    gather of each expert's tokens].  Returns
      counts  [E]    assignments per expert before the capacity drop
      offsets [E+1]  start of each expert's kept rows in the permuted order
      perm_src [N_kept]  the assignment id a held by each permuted row
      slot_pos [T*k] permuted row of each assignment, -1 if dropped
    """
    flat = np.asarray(idx, np.int64).reshape(-1)
    n = flat.shape[0]
    counts = np.zeros(E, np.int64)
    for e in range(E):
        counts[e] = int(np.sum(flat == e))
    kept = counts if C is None else np.minimum(counts, C)
    offsets = np.zeros(E + 1, np.int64)
    offsets[1:] = np.cumsum(kept)
    slot_pos = np.full(n, -1, np.int64)
    perm_src = np.zeros(int(offsets[-1]), np.int64)
    for e in range(E):
        members = np.nonzero(flat == e)[0]          # ascending assignment id
        keep = members[: int(kept[e])]
        slots = offsets[e] + np.arange(keep.shape[0])
        slot_pos[keep] = slots
        perm_src[slots] = keep
    return counts, offsets, perm_src, slot_pos


def gather_rows(x, perm_src, k):
    """x_perm[s] = x[perm_src[s] // k]: each kept assignment's token row."""
    return _f64(x)[np.asarray(perm_src) // k]


# ------------------------------------------------------------------------- experts


def gelu(z):
    """GELU(z) = z * Phi(z) = 0.5 z (1 + erf(z / sqrt 2)) (exact form)."""
    z = _f64(z)
    return 0.5 * z * (1.0 + erf(z / math.sqrt(2.0)))


def relu(z):
    return np.maximum(_f64(z), 0.0)


ACTS = {"relu": relu, "gelu": gelu}


def expert(x_rows, w1_e, w2_e, act):
    """One expert, a feed-forward sub-network E_i(x) = W2_i act(W1_i x) [SGMoE
    "Schlüsselbegriffe"].  x_rows [n, d]; w1_e [f, d]; w2_e [d, f].  Returns (h, y)."""
    h = ACTS[act](_f64(x_rows) @ _f64(w1_e).T)
    y = h @ _f64(w2_e).T
    return h, y


def expert_ffn(x_perm, offsets, w1, w2, act):
    """Apply expert e to its permuted rows [offsets[e], offsets[e+1]).  Returns (h, y_perm)."""
    x_perm = _f64(x_perm)
    n = x_perm.shape[0]
    E, f, d = w1.shape
    h = np.zeros((n, f))
    y = np.zeros((n, d))
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b > a:
            h[a:b], y[a:b] = expert(x_perm[a:b], w1[e], w2[e], act)
    return h, y


def combine(y_perm, slot_pos, gates, T, k):
    """y_t = sum_j G_{t,j} * y_perm[slot_pos[t, j]]; a dropped slot adds nothing
    [SGMoE: y = sum_i G(x)_i E_i(x), computation skipped where G(x)_i = 0]."""
    y_perm = _f64(y_perm)
    y = np.zeros((T, y_perm.shape[1]))
    sp = np.asarray(slot_pos).reshape(T, k)
    for j in range(k):
        keep = sp[:, j] >= 0
        y[keep] += gates[keep, j][:, None] * y_perm[sp[keep, j]]
    return y


# ---------------------------------------------------------------------- whole layer


def route(inp, w):
    """Gating for workload ``w`` on inputs ``inp`` (numpy arrays or CPU torch tensors).  Returns a dict with scores, idx [T,k], gates [T,k], gap [T] and, for
    noisy gating, l, s, importance, load."""
    x = inp["x"]
    bias = inp.get("logit_bias")
    out = {}
    if w.gating == "hierarchical":
        scores = router_logits(x, inp["w_gate"], bias)
        idx, gates, gap = hierarchical_gates(scores, w.groups, w.k_primary, w.k // w.k_primary)
        out.update(scores=scores, idx=idx, gates=gates, gap=gap)
        return out
    if w.gating == "noisy_topk":
        l, s, H = noisy_logits(x, inp["w_gate"], inp["w_noise"], inp["noise"], bias)
        scores = H
        out.update(l=l, s=s)
    else:
        scores = router_logits(x, inp["w_gate"], bias)
    idx = top_k(scores, w.k)
    renorm = True if w.gating == "noisy_topk" else w.renorm
    gates = gate_values(scores, idx, renorm)
    out.update(scores=scores, idx=idx, gates=gates, gap=topk_gap(scores, w.k))
    if w.gating == "noisy_topk":
        G = dense_gates(scores.shape[0], w.E, idx, gates)
        out["importance"] = importance(G)
        if w.k < w.E:
            out["load"] = load(load_probability(out["l"], out["s"], scores, w.k))
    return out


def moe_forward(inp, w):
    """The whole layer, sparse evaluation: route, dispatch with capacity, per-expert FFN on
    the kept rows only, gate-weighted combine."""
    r = route(inp, w)
    T = r["idx"].shape[0]
    C = capacity(w.capacity_factor, T, w.k, w.E)
    counts, offsets, perm_src, slot_pos = dispatch(r["idx"], w.E, C)
    x_perm = gather_rows(inp["x"], perm_src, w.k)
    h, y_perm = expert_ffn(x_perm, offsets, inp["w1"], inp["w2"], w.act)
    gates = r["gates"]
    y = combine(y_perm, slot_pos, gates, T, w.k)
    r.update(C=C, counts=counts, offsets=offsets, perm_src=perm_src, slot_pos=slot_pos,
             x_perm=x_perm, h=h, y_perm=y_perm, y=y)
    return r


def moe_forward_dense(inp, w):
    """The layer by its definition y = sum_i G(x)_i E_i(x) [SGMoE "Methode"]: every expert
    evaluated on every token, weighted by the dense gate matrix (dropped assignments get
    G = 0).  Only for tiny inputs."""
    r = route(inp, w)
    T = r["idx"].shape[0]
    C = capacity(w.capacity_factor, T, w.k, w.E)
    _, _, _, slot_pos = dispatch(r["idx"], w.E, C)
    if w.gating == "hierarchical":
        # the two-level definition, dense; then dropped assignments get 0
        G = hierarchical_dense_gates(r["scores"], w.groups, w.k_primary, w.k // w.k_primary)
        keep = np.ones((T, w.E))
        sp = slot_pos.reshape(T, w.k)
        for j in range(w.k):
            drop = sp[:, j] < 0
            keep[np.nonzero(drop)[0], r["idx"][drop, j]] = 0.0
        G = G * keep
    else:
        G = dense_gates(T, w.E, r["idx"], r["gates"], slot_pos)
    x = _f64(inp["x"])
    y = np.zeros((T, x.shape[1]))
    for e in range(w.E):
        _, ye = expert(x, inp["w1"][e], inp["w2"][e], w.act)
        y += G[:, e:e + 1] * ye
    return y


def moe_forward_rows(inp, w, rows, idx=None, gates=None):
    """Layer outputs for the token rows ``rows`` only.

    Routing and dispatch run over all tokens (capacity depends on every token's choice);
    the expert FFN runs only for the requested tokens' kept assignments.  ``idx``/``gates``
    may override the routing (e.g. to follow another side's choice at near ties).
    Returns (y_rows [len(rows), d], routing dict)."""
    if idx is None:
        r = route(inp, w)
        idx, gates = r["idx"], r["gates"]
    else:
        r = {"idx": idx, "gates": gates}
    T = idx.shape[0]
    C = capacity(w.capacity_factor, T, w.k, w.E)
    counts, offsets, perm_src, slot_pos = dispatch(idx, w.E, C)
    x = inp["x"]
    sp = slot_pos.reshape(T, w.k)
    y = np.zeros((len(rows), x.shape[1]))
    for n, t in enumerate(rows):
        xt = _f64(x[t:t + 1])
        for j in range(w.k):
            if sp[t, j] >= 0:
                e = int(idx[t, j])
                _, ye = expert(xt, inp["w1"][e], inp["w2"][e], w.act)
                y[n] += gates[t, j] * ye[0]
    r.update(C=C, counts=counts, offsets=offsets, perm_src=perm_src, slot_pos=slot_pos)
    return y, r
