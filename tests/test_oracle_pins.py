"""Pins of the CPU oracle to things other than itself: hand-worked examples
(tests/golden/), library routines (torch.nn.functional, torch.topk, scipy.stats),
closed forms, invariants and brute force on tiny inputs.

Each test names the page section it pins.  None of them re-types the oracle's formula:
the expected values come from a derivation by hand or a different routine.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from scipy.stats import norm

from oracle import moe_oracle as orc
import workloads

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ------------------------------------------------------------------ router logits


def test_router_logits_hand():
    # x.W_g with W_g stored one row per expert; integers, worked by hand.
    x = np.array([[1.0, 2.0], [3.0, 4.0]])
    wg = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]])        # [E=3, d=2]
    assert np.array_equal(orc.router_logits(x, wg), [[1, 2, 3], [3, 4, 7]])
    bias = np.array([0.5, 0.0, -1.0])
    assert np.array_equal(orc.router_logits(x, wg, bias), [[1.5, 2, 2], [3.5, 4, 6]])


def test_router_logits_matches_torch_linear():
    g = np.random.default_rng(1)
    x, wg = g.standard_normal((7, 5)), g.standard_normal((3, 5))
    ref = F.linear(torch.from_numpy(x), torch.from_numpy(wg)).numpy()
    assert np.allclose(orc.router_logits(x, wg), ref, rtol=0, atol=1e-13)


# ------------------------------------------------------------------ gating (top-k)


@pytest.mark.parametrize("case", _gold("gating_hand.json")["cases"])
def test_gating_hand_cases(case):
    """Softmax(KeepTopK) and the Switch top-1 probability on hand-worked logits."""
    scores = np.log(np.array([case["q"]], np.float64))
    idx = orc.top_k(scores, case["k"])
    assert idx[0].tolist() == case["idx"]
    gates = orc.gate_values(scores, idx, case["renorm"])[0]
    want = [n / d for n, d in case["gates"]]
    assert np.allclose(gates, want, rtol=1e-14, atol=0)


def test_top_k_brute_force_with_ties():
    """Lowest-index tie break: brute force over every row of small integer scores."""
    g = np.random.default_rng(2)
    for E in range(1, 6):
        rows = np.array(list(itertools.product(range(3), repeat=E)), np.float64)
        for k in range(1, E + 1):
            got = orc.top_k(rows, k)
            for r, row in enumerate(rows):
                want = sorted(range(E), key=lambda i: (-row[i], i))[:k]
                assert got[r].tolist() == want
    v = g.standard_normal((50, 9))
    assert orc.top_k(v, 3).tolist() == torch.topk(torch.from_numpy(v), 3).indices.tolist()


def test_gates_match_torch_softmax_topk():
    """Library cross-check on tie-free rows: Switch gate = topk of torch.softmax;
    renormalised gate = torch.softmax over the top-k logits."""
    g = np.random.default_rng(3)
    l = g.standard_normal((40, 12)) * 2
    lt = torch.from_numpy(l)
    p_top1, i_top1 = torch.topk(torch.softmax(lt, -1), 1)
    idx = orc.top_k(l, 1)
    assert idx.tolist() == i_top1.tolist()
    assert np.allclose(orc.gate_values(l, idx, False), p_top1.numpy(), rtol=1e-14)
    v4, i4 = torch.topk(lt, 4)
    idx4 = orc.top_k(l, 4)
    assert idx4.tolist() == i4.tolist()
    assert np.allclose(orc.gate_values(l, idx4, True), torch.softmax(v4, -1).numpy(),
                       rtol=1e-14)


def test_keep_topk_softmax_equals_renormalised_full_softmax():
    """Softmax(KeepTopK(v,k)) restricted to the chosen experts equals the full softmax's
    chosen probabilities divided by their sum (an identity of exp)."""
    g = np.random.default_rng(4)
    v = g.standard_normal((30, 10)) * 3
    idx = orc.top_k(v, 3)
    rows = np.arange(30)[:, None]
    p = np.exp(v) / np.exp(v).sum(1, keepdims=True)
    want = p[rows, idx] / p[rows, idx].sum(1, keepdims=True)
    assert np.allclose(orc.gate_values(v, idx, True), want, rtol=1e-13)
    assert np.allclose(orc.gate_values(v, idx, True).sum(1), 1.0, rtol=0, atol=1e-14)


def test_single_expert_gate_is_one():
    v = np.random.default_rng(5).standard_normal((8, 1))
    idx = orc.top_k(v, 1)
    assert np.all(idx == 0)
    assert np.array_equal(orc.gate_values(v, idx, True), np.ones((8, 1)))
    assert np.array_equal(orc.gate_values(v, idx, False), np.ones((8, 1)))


def test_topk_gap_hand():
    v = np.array([[3.0, 1.0, 2.0, 2.0]])
    assert orc.topk_gap(v, 1)[0] == 1.0
    assert orc.topk_gap(v, 2)[0] == 0.0
    assert orc.topk_gap(v, 3)[0] == 1.0
    assert np.isinf(orc.topk_gap(v, 4)[0])


# ------------------------------------------------------------------ noisy gating


def test_softplus_closed_forms():
    z = np.array([-800.0, -30.0, -1.0, 0.0, 1.0, 30.0, 800.0])
    got = orc.softplus(z)
    assert got[3] == math.log(2.0)
    assert got[-1] == 800.0 and got[-2] == pytest.approx(30.0, abs=1e-12)
    assert got[0] == 0.0 or got[0] < 1e-300
    assert got[1] == pytest.approx(math.exp(-30.0), rel=1e-12)
    assert np.allclose(got[2:5], np.log1p(np.exp(z[2:5])), rtol=1e-15)
    mid = np.linspace(-20, 20, 101)
    assert np.allclose(orc.softplus(mid), F.softplus(torch.from_numpy(mid)).numpy(),
                       rtol=1e-14, atol=1e-300)


def _noisy_hand():
    gd = _gold("noisy_hand.json")
    s = np.array(gd["s_target"])
    w_noise = np.log(np.expm1(s))[:, None]            # inverse softplus, so x.W_noise gives s
    return gd, np.array(gd["x"]), np.array(gd["w_gate"]), w_noise, np.array(gd["noise"])


def test_noisy_logits_hand():
    gd, x, wg, wn, n = _noisy_hand()
    l, s, H = orc.noisy_logits(x, wg, wn, n)
    assert np.array_equal(l, [[0.0, 0.0, 0.0]])
    assert np.allclose(s[0], gd["s_target"], rtol=1e-14)
    assert np.allclose(H[0], gd["H"], rtol=1e-14)


@pytest.mark.parametrize("k", [1, 2])
def test_noisy_gate_load_importance_hand(k):
    gd, x, wg, wn, n = _noisy_hand()
    case = gd["k%d" % k]
    l, s, H = orc.noisy_logits(x, wg, wn, n)
    idx = orc.top_k(H, k)
    assert idx[0].tolist() == case["idx"]
    G = orc.dense_gates(1, 3, idx, orc.gate_values(H, idx, True))
    if k == 1:
        assert np.array_equal(G[0], case["G_dense"])
    else:
        u = np.array(case["G_chosen_unnormalised"])
        assert np.allclose(G[0, :2], u / u.sum(), rtol=1e-14) and G[0, 2] == 0.0
    assert np.allclose(orc.kth_excluding(H, k)[0], case["kth_excluding"], rtol=1e-14)
    P = orc.load_probability(l, s, H, k)
    assert np.allclose(P[0], norm.cdf(case["phi_args"]), rtol=1e-13)
    assert np.allclose(orc.importance(G), G.sum(0))
    assert np.allclose(orc.load(P), norm.cdf(case["phi_args"]), rtol=1e-13)


def test_noise_zero_reduces_to_clean_logits():
    g = np.random.default_rng(6)
    x, wg, wn = g.standard_normal((9, 4)), g.standard_normal((5, 4)), g.standard_normal((5, 4))
    l, s, H = orc.noisy_logits(x, wg, wn, np.zeros((9, 5)))
    assert np.array_equal(H, l)
    assert np.all(s > 0)


def test_kth_excluding_brute_force():
    """Closed form vs the definition (k-th largest of the other experts' H), with ties."""
    g = np.random.default_rng(7)
    for E in (2, 3, 5, 8):
        H = np.concatenate([g.integers(0, 3, (40, E)).astype(np.float64),
                            g.standard_normal((40, E))])
        for k in range(1, E):
            got = orc.kth_excluding(H, k)
            for t in range(H.shape[0]):
                for i in range(E):
                    others = sorted((H[t, j] for j in range(E) if j != i), reverse=True)
                    assert got[t, i] == others[k - 1]


def test_std_normal_cdf_matches_scipy():
    z = np.linspace(-9, 9, 181)
    assert np.allclose(orc.std_normal_cdf(z), norm.cdf(z), rtol=1e-13, atol=1e-300)
    assert orc.std_normal_cdf(0.0) == 0.5


def test_load_probability_in_unit_interval():
    g = np.random.default_rng(8)
    x, wg, wn = g.standard_normal((50, 6)), g.standard_normal((7, 6)), g.standard_normal((7, 6))
    l, s, H = orc.noisy_logits(x, wg, wn, g.standard_normal((50, 7)))
    P = orc.load_probability(l, s, H, 2)
    assert np.all(P >= 0) and np.all(P <= 1)


# ------------------------------------------------------------------ capacity, dispatch


def test_capacity_hand():
    for c in _gold("dispatch_hand.json")["capacity"]:
        assert orc.capacity(c["cf"], c["T"], c["k"], c["E"]) == c["C"], c


@pytest.mark.parametrize("case", _gold("dispatch_hand.json")["cases"])
def test_dispatch_hand(case):
    counts, offsets, perm_src, slot_pos = orc.dispatch(np.array(case["idx"]), case["E"], case["C"])
    assert counts.tolist() == case["counts"]
    assert offsets.tolist() == case["offsets"]
    assert perm_src.tolist() == case["perm_src"]
    assert slot_pos.tolist() == case["slot_pos"]


def test_dispatch_invariants_brute_force():
    """Bijection on kept slots, counts equal a brute-force tally, no expert above C,
    and the kept set of each expert is its first C assignments in token order."""
    g = np.random.default_rng(9)
    for (T, E, k, C) in [(200, 7, 2, None), (200, 7, 2, 30), (97, 4, 3, 5), (64, 16, 1, 1)]:
        idx = np.stack([g.permutation(E)[:k] for _ in range(T)])
        counts, offsets, perm_src, slot_pos = orc.dispatch(idx, E, C)
        tally = [0] * E
        for a, e in enumerate(idx.reshape(-1)):
            tally[e] += 1
        assert counts.tolist() == tally
        kept = slot_pos >= 0
        assert sorted(slot_pos[kept].tolist()) == list(range(int(offsets[-1])))
        assert np.array_equal(perm_src[slot_pos[kept]], np.nonzero(kept)[0])
        for e in range(E):
            n_e = offsets[e + 1] - offsets[e]
            assert n_e == (tally[e] if C is None else min(tally[e], C))
            members = [a for a, ee in enumerate(idx.reshape(-1)) if ee == e]
            assert perm_src[offsets[e]:offsets[e + 1]].tolist() == members[:n_e]


# ------------------------------------------------------------------ experts, layer


def _tiny_inputs(T, d, f, E, seed, noisy=False):
    g = np.random.default_rng(seed)
    inp = {"x": g.standard_normal((T, d)), "w_gate": g.standard_normal((E, d)) / math.sqrt(d),
           "w1": g.standard_normal((E, f, d)) / math.sqrt(d),
           "w2": g.standard_normal((E, d, f)) / math.sqrt(f)}
    if noisy:
        inp["w_noise"] = g.standard_normal((E, d)) / math.sqrt(d)
        inp["noise"] = g.standard_normal((T, E))
    return inp


def test_gelu_matches_torch_exact_gelu():
    z = np.linspace(-8, 8, 321)
    assert np.allclose(orc.gelu(z), F.gelu(torch.from_numpy(z), approximate="none").numpy(),
                       rtol=1e-14, atol=1e-300)
    assert orc.gelu(1.0) == pytest.approx(norm.cdf(1.0), rel=1e-15)


@pytest.mark.parametrize("act", ["relu", "gelu"])
def test_single_expert_layer_is_dense_ffn(act):
    """E=1, k=1, no capacity: the layer is one dense FFN (torch.nn.functional)."""
    inp = _tiny_inputs(33, 12, 20, 1, 10)
    for gating, renorm in [("softmax_topk", True), ("softmax_topk", False)]:
        w = workloads.Workload("t", T=33, d_model=12, d_ff=20, E=1, k=1, gating=gating,
                               renorm=renorm, act=act, dtype="f32")
        y = orc.moe_forward(inp, w)["y"]
        xt = torch.from_numpy(inp["x"])
        h = F.linear(xt, torch.from_numpy(inp["w1"][0]))
        h = F.relu(h) if act == "relu" else F.gelu(h, approximate="none")
        ref = F.linear(h, torch.from_numpy(inp["w2"][0])).numpy()
        assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("cfg", [
    dict(T=48, E=6, k=2, gating="softmax_topk", renorm=True, cf=None),
    dict(T=48, E=6, k=2, gating="softmax_topk", renorm=True, cf=0.5),
    dict(T=64, E=5, k=1, gating="softmax_topk", renorm=False, cf=1.0),
    dict(T=40, E=8, k=4, gating="noisy_topk", renorm=True, cf=None),
    dict(T=40, E=8, k=3, gating="noisy_topk", renorm=True, cf=0.75),
])
def test_sparse_equals_dense_definition(cfg):
    """y = sum_i G(x)_i E_i(x) evaluated densely equals the sparse dispatch path."""
    inp = _tiny_inputs(cfg["T"], 10, 14, cfg["E"], 11, noisy=cfg["gating"] == "noisy_topk")
    w = workloads.Workload("t", T=cfg["T"], d_model=10, d_ff=14, E=cfg["E"], k=cfg["k"],
                           gating=cfg["gating"], renorm=cfg["renorm"],
                           capacity_factor=cfg["cf"], act="gelu", dtype="f32")
    sparse = orc.moe_forward(inp, w)
    dense = orc.moe_forward_dense(inp, w)
    assert np.allclose(sparse["y"], dense, rtol=0, atol=1e-12)
    rows = [0, 5, cfg["T"] - 1]
    y_rows, _ = orc.moe_forward_rows(inp, w, rows)
    assert np.allclose(y_rows, sparse["y"][rows], rtol=0, atol=1e-12)


def test_dropped_tokens_output_zero():
    """E=1, k=1, C = ceil(0.5*T): tokens past capacity give exactly 0; the rest are the
    dense FFN."""
    T = 21
    inp = _tiny_inputs(T, 8, 16, 1, 12)
    w = workloads.Workload("t", T=T, d_model=8, d_ff=16, E=1, k=1, capacity_factor=0.5,
                           act="relu", dtype="f32")
    r = orc.moe_forward(inp, w)
    C = r["C"]
    assert C == 11
    assert np.all(r["y"][C:] == 0.0)
    assert np.all(np.abs(r["y"][:C]).sum(1) > 0)


def test_importance_sums_to_T_and_gates_sum_to_one():
    T = 64
    inp = _tiny_inputs(T, 10, 12, 8, 13, noisy=True)
    w = workloads.Workload("t", T=T, d_model=10, d_ff=12, E=8, k=3, gating="noisy_topk",
                           dtype="f32")
    r = orc.route(inp, w)
    assert np.allclose(r["gates"].sum(1), 1.0, atol=1e-14)
    assert r["importance"].sum() == pytest.approx(T, rel=1e-14)
    assert r["load"].shape == (8,) and np.all(r["load"] >= 0) and np.all(r["load"] <= T)


# ------------------------------------------------------------- hierarchical gating


@pytest.mark.parametrize("case", _gold("hierarchical_hand.json")["cases"])
def test_hierarchical_gating_hand_cases(case):
    """Two-level Softmax(KeepTopK) on hand-worked logits (ties at both levels)."""
    l = np.log(np.array([case["q"]], np.float64))
    idx, gates, _ = orc.hierarchical_gates(l, case["a"], case["k_primary"], case["k_group"])
    assert idx[0].tolist() == case["idx"]
    assert np.allclose(gates[0], [n / d for n, d in case["gates"]], rtol=1e-14, atol=0)


def _hier_brute(row, a, k1, k2):
    """Pure-Python loops: sort groups, then each chosen group's experts, by (-score,
    index); shares from math.exp over the kept entries of each level."""
    b = (len(row) - a) // a
    prim = [row[i] for i in range(a)]
    groups = sorted(range(a), key=lambda i: (-float(np.float32(prim[i])), i))[:k1]
    zp = sum(math.exp(prim[i] - prim[groups[0]]) for i in groups)
    idx, gates = [], []
    for gi in groups:
        sec = [row[a + gi * b + j] for j in range(b)]
        chosen = sorted(range(b), key=lambda j: (-float(np.float32(sec[j])), j))[:k2]
        zs = sum(math.exp(sec[j] - sec[chosen[0]]) for j in chosen)
        for j in chosen:
            idx.append(gi * b + j)
            gates.append(math.exp(prim[gi] - prim[groups[0]]) / zp *
                         math.exp(sec[j] - sec[chosen[0]]) / zs)
    return idx, gates


@pytest.mark.parametrize("a,b,k1,k2", [(4, 3, 2, 2), (3, 5, 1, 3), (5, 2, 3, 1), (2, 6, 2, 4)])
def test_hierarchical_gating_brute_force(a, b, k1, k2):
    g = np.random.default_rng(20 + a * b)
    # coarse values make ties at both levels frequent
    l = np.round(g.standard_normal((60, a + a * b)) * 2) / 2
    idx, gates, _ = orc.hierarchical_gates(l, a, k1, k2)
    for t in range(l.shape[0]):
        bi, bg = _hier_brute(l[t], a, k1, k2)
        assert idx[t].tolist() == bi
        assert np.allclose(gates[t], bg, rtol=1e-13, atol=0)
    assert np.allclose(gates.sum(1), 1.0, rtol=0, atol=1e-14)


def test_hierarchical_one_group_is_flat_topk():
    """One group: the primary gate is 1 and the layer is flat top-k over its experts
    (torch.topk, then torch.softmax over the kept logits)."""
    g = np.random.default_rng(30)
    l = g.standard_normal((40, 1 + 9))
    idx, gates, _ = orc.hierarchical_gates(l, 1, 1, 3)
    v, i = torch.topk(torch.from_numpy(l[:, 1:]), 3)
    assert idx.tolist() == i.tolist()
    assert np.allclose(gates, torch.softmax(v, -1).numpy(), rtol=1e-13)


def test_hierarchical_single_expert_groups_is_flat_topk_over_groups():
    """Groups of one expert: the secondary gate is 1 and the layer is flat top-k over the
    primary logits."""
    g = np.random.default_rng(31)
    a = 7
    l = np.concatenate([g.standard_normal((40, a)), g.standard_normal((40, a))], axis=1)
    idx, gates, _ = orc.hierarchical_gates(l, a, 3, 1)
    v, i = torch.topk(torch.from_numpy(l[:, :a]), 3)
    assert idx.tolist() == i.tolist()
    assert np.allclose(gates, torch.softmax(v, -1).numpy(), rtol=1e-13)


def _hier_inputs(T, d, f, a, b, seed):
    inp = _tiny_inputs(T, d, f, a * b, seed)
    g = np.random.default_rng(seed + 1000)
    inp["w_gate"] = g.standard_normal((a + a * b, d)) / math.sqrt(d)
    return inp


@pytest.mark.parametrize("cf", [None, 0.5])
def test_hierarchical_sparse_equals_dense_definition(cf):
    """y = sum_i G_p(x)_i sum_j G_i(x)_j E_ij(x) evaluated densely (every group's
    secondary gate) equals the sparse dispatch path, also with capacity drops."""
    a, b = 3, 4
    inp = _hier_inputs(48, 10, 14, a, b, 40)
    w = workloads.Workload("h", T=48, d_model=10, d_ff=14, E=a * b, k=4, gating="hierarchical",
                           groups=a, k_primary=2, capacity_factor=cf, act="gelu", dtype="f32")
    sparse = orc.moe_forward(inp, w)
    dense = orc.moe_forward_dense(inp, w)
    assert np.allclose(sparse["y"], dense, rtol=0, atol=1e-12)
    if cf is not None:
        assert int(sparse["offsets"][-1]) < 48 * 4   # some assignments were dropped
    rows = [0, 7, 47]
    y_rows, _ = orc.moe_forward_rows(inp, w, rows)
    assert np.allclose(y_rows, sparse["y"][rows], rtol=0, atol=1e-12)


def test_oracle_and_library_share_no_code():
    """The oracle never imports the CUDA library's package, and the package never
    imports the oracle."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for fn in os.listdir(os.path.join(root, "oracle")):
        if fn.endswith(".py"):
            assert "sparsely_gated_mixture_moe_b200" not in open(os.path.join(root, "oracle", fn)).read()
    pkg = os.path.join(root, "sparsely_gated_mixture_moe_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in src and "from oracle" not in src, fn
