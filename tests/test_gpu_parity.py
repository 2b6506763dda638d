"""Parity of the CUDA path with the CPU oracle, element by element, on seeded inputs.

Small cases (the oracle finishes in seconds) cover every workload's shape family at a
reduced token count, several 128-row tiles with ragged tails, each N-tile width of the
grouped GEMM, capacity stress, and the degenerate cases (one expert, k = E, one token,
no tokens, T not a multiple of the tile).  The full-size cases run the exact workloads
the benchmark times and compare sampled outputs plus everything that is cheap to check
everywhere (choices, gates, the permutation, counts)."""
import numpy as np
import pytest
import torch

import workloads
from workloads import Workload
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu

W = workloads.WORKLOADS
SMALL = {
    "tiny": W["tiny"],
    "switch_T2048": W["switch"].scaled(T=2048),
    "noisy_T1024": W["noisy"].scaled(T=1024),
    "gshard_T1024": W["gshard"].scaled(T=1024),
    "zipf_T2048": W["zipf"].scaled(T=2048),
    "multitile_T4096": Workload("mt", T=4096, d_model=256, d_ff=512, E=16, k=2, act="gelu"),
    "bn128_T1000": Workload("b128", T=1000, d_model=384, d_ff=640, E=12, k=3, act="relu"),
    "bn64_T777": Workload("b64", T=777, d_model=448, d_ff=192, E=5, k=2, act="gelu"),
    "cap0.25": Workload("c25", T=1024, d_model=128, d_ff=256, E=8, k=2, capacity_factor=0.25),
    "cap0.5_switch": Workload("c50", T=1024, d_model=128, d_ff=256, E=8, k=1, renorm=False,
                              capacity_factor=0.5, act="gelu"),
    "cap1.0": Workload("c100", T=1024, d_model=128, d_ff=256, E=8, k=2, capacity_factor=1.0),
    "noisy_small_E": Workload("nz", T=600, d_model=128, d_ff=128, E=12, k=3, gating="noisy_topk"),
    "f32_noisy": Workload("f32n", T=300, d_model=64, d_ff=96, E=10, k=3, gating="noisy_topk",
                          dtype="f32"),
    "f32_switch_cap": Workload("f32s", T=257, d_model=32, d_ff=64, E=6, k=1, renorm=False,
                               capacity_factor=0.75, act="gelu", dtype="f32"),
    "one_expert": Workload("e1", T=300, d_model=128, d_ff=128, E=1, k=1),
    "k_equals_E": Workload("kE", T=200, d_model=64, d_ff=128, E=4, k=4, act="gelu"),
    "one_token": Workload("t1", T=1, d_model=64, d_ff=64, E=8, k=2),
    "E8_bf16_pad": Workload("e8", T=500, d_model=64, d_ff=64, E=8, k=2),
    "f16_hidden_multitile": Workload("h16", T=3000, d_model=192, d_ff=384, E=6, k=2, act="gelu",
                                     hidden_f16=True, capacity_factor=0.9),
    # k = 8: the router's longest top lists (two column groups of gate warps)
    "k8_E32": Workload("k8", T=1500, d_model=128, d_ff=128, E=32, k=8, act="relu"),
    # the largest supported expert counts: fp32 E = 1024 (the one-launch permutation's
    # biggest shared-memory footprint) and bf16 E = 256 with k = 8
    "f32_E1024": Workload("e1024", T=2048, d_model=32, d_ff=32, E=1024, k=2, dtype="f32"),
    "E256_k8": Workload("e256k8", T=1200, d_model=128, d_ff=128, E=256, k=8, act="gelu",
                        capacity_factor=2.0),
    # noisy gating with capacity drops (Importance still sums the gates before the drop)
    "noisy_capacity": Workload("nzc", T=900, d_model=128, d_ff=128, E=16, k=2,
                               gating="noisy_topk", capacity_factor=0.5),
    # hierarchical (two-level) gating: 8 groups of 16 keeping 2 x 2; one kept group of
    # 16 groups with capacity drops; 1 x 3 in fp32; 2 x 4 and 4 x 2 (the longest lists
    # per level, k = 8)
    "hier_8x16_k2x2": Workload("h1", T=1500, d_model=128, d_ff=128, E=128, k=4,
                               gating="hierarchical", groups=8, k_primary=2, act="gelu"),
    "hier_16x4_k1x1_cap": Workload("h2", T=1000, d_model=64, d_ff=128, E=64, k=1,
                                   gating="hierarchical", groups=16, k_primary=1,
                                   capacity_factor=1.0),
    "hier_f32_3x4_k1x3": Workload("h3", T=300, d_model=64, d_ff=64, E=12, k=3,
                                  gating="hierarchical", groups=3, k_primary=1, dtype="f32"),
    "hier_4x16_k2x4": Workload("h4", T=700, d_model=128, d_ff=64, E=64, k=8,
                               gating="hierarchical", groups=4, k_primary=2, act="relu"),
    "hier_8x8_k4x2": Workload("h5", T=700, d_model=128, d_ff=64, E=64, k=8,
                              gating="hierarchical", groups=8, k_primary=4, act="relu"),
    # the router's gate splits the groups over its column groups: 32 primary columns (two
    # 16-column slices) with four groups to a slice; two groups of 64 (each over four
    # slices, most column groups idle); groups of 12 straddling slices with three of five
    # kept; 128-token tiles (more than 74 of them) instead of 64-token ones
    "hier_32x4_k2x1": Workload("h6", T=1000, d_model=128, d_ff=64, E=128, k=2,
                               gating="hierarchical", groups=32, k_primary=2, act="relu"),
    "hier_2x64_k1x4": Workload("h7", T=333, d_model=64, d_ff=64, E=128, k=4,
                               gating="hierarchical", groups=2, k_primary=1, act="gelu"),
    "hier_5x12_k3x1": Workload("h8", T=517, d_model=64, d_ff=64, E=60, k=3,
                               gating="hierarchical", groups=5, k_primary=3, act="relu"),
    "hier_full_tiles_T10000": Workload("h9", T=10000, d_model=128, d_ff=64, E=64, k=4,
                                       gating="hierarchical", groups=8, k_primary=2,
                                       act="relu"),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_steps_and_forward_small(name):
    w = SMALL[name]
    inp = workloads.make_inputs(w)
    dev = H.to_device(inp)
    g = H.run_steps(w, dev)
    assert g["device_error"] == 0
    rep = {}
    idx, gates = H.check_route(w, inp, g, rep)
    n = H.check_permute(w, inp, g, rep)
    H.check_ffn(w, inp, g, n, rep)
    H.check_combine(w, g, rep)
    H.check_end_to_end(w, inp, g, idx, gates, rep)
    H.check_gather_path(w, g, rep)
    f = H.run_forward(w, dev)
    assert f["device_error"] == 0
    # the fused call runs the same kernels: identical results
    assert torch.equal(f["topk_idx"], g["topk_idx"])
    assert torch.equal(f["counts"], g["counts"])
    assert torch.equal(f["y"], g["y"])
    print(name, rep)


def _random_cases(n=16, seed=2024):
    """Seeded random small layers: dtype, expert count (1 to 256), k (up to 8, <= E),
    gating, capacity, activation, widths and token counts drawn independently, so that
    shapes no hand-written case names still meet the oracle.  A Switch-style top-1 gate
    (renorm off) stores h in fp16, as the Switch workload does (its gates vary too much for
    one bf16 rounding of h within the bar)."""
    rng = np.random.default_rng(seed)
    cases = {}
    for i in range(n):
        dtype = "f32" if i % 5 == 4 else "bf16"
        E = int(rng.choice([1, 2, 3, 5, 8, 13, 16, 32, 64, 100, 256]))
        k = int(rng.integers(1, min(E, 8) + 1))
        gating = "noisy_topk" if rng.random() < 0.3 else "softmax_topk"
        renorm = True if (gating == "noisy_topk" or k > 1) else bool(rng.random() < 0.5)
        if dtype == "bf16":
            d = int(rng.choice([64, 128, 192, 256, 512]))
            f = int(rng.choice([64, 128, 192, 320, 512, 1024]))
        else:
            d = int(rng.choice([8, 24, 64, 96]))
            f = int(rng.choice([4, 12, 64, 100]))
        T = int(rng.integers(1, 2500))
        cf = None if rng.random() < 0.5 else float(rng.choice([0.5, 0.8, 1.0, 1.25, 2.0]))
        act = "gelu" if rng.random() < 0.5 else "relu"
        hidden_f16 = dtype == "bf16" and (not renorm or rng.random() < 0.3)
        name = "rand%02d_%s_T%d_E%d_k%d_%s" % (i, dtype, T, E, k, gating.split("_")[0])
        cases[name] = Workload("r%02d" % i, T=T, d_model=d, d_ff=f, E=E, k=k, gating=gating,
                               renorm=renorm, capacity_factor=cf, act=act, dtype=dtype,
                               hidden_f16=hidden_f16, seed=100 + i)
    return cases


RANDOM = _random_cases()


@pytest.mark.parametrize("name", list(RANDOM))
def test_steps_and_forward_random_shapes(name):
    w = RANDOM[name]
    inp = workloads.make_inputs(w)
    dev = H.to_device(inp)
    g = H.run_steps(w, dev)
    assert g["device_error"] == 0
    rep = {}
    idx, gates = H.check_route(w, inp, g, rep)
    n = H.check_permute(w, inp, g, rep)
    H.check_ffn(w, inp, g, n, rep)
    H.check_combine(w, g, rep)
    H.check_end_to_end(w, inp, g, idx, gates, rep)
    H.check_gather_path(w, g, rep)
    f = H.run_forward(w, dev)
    assert f["device_error"] == 0
    assert torch.equal(f["y"], g["y"])
    print(name, rep)


def test_empty_batch():
    w = Workload("t0", T=0, d_model=64, d_ff=64, E=4, k=2, gating="noisy_topk")
    inp = workloads.make_inputs(w)
    dev = H.to_device(inp)
    g = H.run_steps(w, dev)
    assert g["device_error"] == 0
    assert g["counts"].tolist() == [0] * 4
    assert g["offsets"].tolist() == [0] * 5
    assert g["importance"].tolist() == [0.0] * 4 and g["load"].tolist() == [0.0] * 4


def test_deterministic_repeat():
    w = SMALL["noisy_T1024"]
    dev = H.to_device(workloads.make_inputs(w))
    a, b = H.run_steps(w, dev), H.run_steps(w, dev)
    for key in ("topk_idx", "topk_gate", "counts", "slot_pos", "y", "importance", "load"):
        assert torch.equal(a[key], b[key]), key


def test_bad_expert_index_sets_error_and_drops():
    """An out-of-range index fed to moe_permute is reported through the device error
    word and treated as dropped; nothing else changes."""
    import sparsely_gated_mixture_moe_b200 as moe
    w = Workload("bad", T=64, d_model=64, d_ff=64, E=4, k=2)
    cfg = H.config_of(w)
    inp = workloads.make_inputs(w)
    x = inp["x"].cuda()
    idx = torch.tensor([[0, 1]] * 64, dtype=torch.int32)
    idx[5, 1] = 7
    idx[9, 0] = -3
    ws = moe.workspace(cfg)
    counts = torch.empty(4, dtype=torch.int32, device="cuda")
    offsets = torch.empty(5, dtype=torch.int32, device="cuda")
    perm_src = torch.empty(128, dtype=torch.int32, device="cuda")
    slot_pos = torch.empty(128, dtype=torch.int32, device="cuda")
    x_perm = torch.empty(128, 64, dtype=torch.bfloat16, device="cuda")
    moe.moe_permute(cfg, idx.cuda(), x, counts, offsets, perm_src, slot_pos, x_perm, ws)
    err = moe.moe_get_error(ws)
    assert err == 1
    assert moe.moe_get_error(ws) == 0  # cleared by the read
    sp = slot_pos.cpu().numpy()
    assert sp[5 * 2 + 1] == -1 and sp[9 * 2 + 0] == -1
    assert counts.cpu().tolist() == [63, 63, 0, 0]


def test_bad_offsets_set_error():
    """Offsets that are not non-decreasing make moe_expert_ffn skip its work and report
    MOE_DEVERR_OFFSETS instead of reading or writing out of range."""
    import sparsely_gated_mixture_moe_b200 as moe
    w = Workload("off", T=64, d_model=64, d_ff=64, E=4, k=1)
    cfg = H.config_of(w)
    inp = H.to_device(workloads.make_inputs(w))
    ws = moe.workspace(cfg)
    offsets = torch.tensor([0, 30, 10, 50, 64], dtype=torch.int32, device="cuda")
    h = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_ffn(cfg, inp["x"], offsets, inp["w1"], inp["w2"], h, y, ws)
    assert moe.moe_get_error(ws) & 2
    offsets = torch.tensor([0, 10, 20, 30, 65], dtype=torch.int32, device="cuda")  # past T*k
    moe.moe_expert_ffn(cfg, inp["x"], offsets, inp["w1"], inp["w2"], h, y, ws)
    assert moe.moe_get_error(ws) & 2


FULL = {name: W[name] for name in ("switch", "noisy", "gshard", "zipf")}
# More assignments (200,000) than one permutation launch can keep resident on a B200
# (1024 per block, one block per SM): moe_permute takes its three-kernel path here.
FULL["three_kernel_permute_T200k"] = Workload("t200k", T=200_000, d_model=64, d_ff=128, E=8, k=1,
                                              renorm=False, capacity_factor=1.0, act="relu")
# Router on 128-token tiles with several tiles per CTA (more than 74 tiles): noisy gating
# with its two products in one TMEM buffer, and k = 8 with two gate column groups.
FULL["noisy_full_tiles_T20000"] = W["noisy"].scaled(T=20_000)
FULL["k8_full_tiles_T12000"] = Workload("k8f", T=12_000, d_model=256, d_ff=256, E=64, k=8,
                                        act="gelu", capacity_factor=1.5)
# just past the half-tile threshold (75 tiles of 128 > 148 / 2): 128-token tiles with a
# ragged last tile
FULL["noisy_full_tiles_ragged_T9473"] = W["noisy"].scaled(T=9_473)
# hierarchical MoE at the noisy workload's size: 8 groups of 16 experts, 2 groups and 2
# experts per group kept ("MoE-H" keeps 2 per level)
FULL["hierarchical_T8192"] = Workload("hier", T=8192, d_model=512, d_ff=1024, E=128, k=4,
                                      gating="hierarchical", groups=8, k_primary=2, act="relu")


# workloads whose every expert row and every token the fp64 oracle checks at full size
# (155 and 69 GFLOP); the others are sampled
FULL_EVERY_ROW = {"switch", "noisy"}


def sampled_rows(off, rng, extra=48):
    """Every expert's first and last kept row, one random row of each of its 128-row
    tiles, plus `extra` random rows."""
    rows = set()
    n = int(off[-1])
    for e in range(len(off) - 1):
        a, b = int(off[e]), int(off[e + 1])
        if b <= a:
            continue
        rows.update((a, b - 1))
        for t0 in range(a, b, 128):
            rows.add(int(rng.integers(t0, min(t0 + 128, b))))
    rows.update(rng.choice(n, size=min(n, extra), replace=False).tolist())
    return sorted(rows)


@pytest.mark.parametrize("name", list(FULL))
def test_full_size_sampled(name):
    """The benchmark's workloads at full size, in the launch configuration the benchmark
    times.  Choices, gates, importance/load and the whole permutation are checked on
    every token.  On the Switch and noisy workloads every expert row (h, y_perm) and every
    token of the layer output are checked; on the others every expert's first and last
    kept row, one row of each of its 128-row tiles, and 512 tokens of the output."""
    w = FULL[name]
    inp = workloads.make_inputs(w)
    dev = H.to_device(inp)
    g = H.run_steps(w, dev)
    assert g["device_error"] == 0
    rep = {}
    idx, gates = H.check_route(w, inp, g, rep)
    n = H.check_permute(w, inp, g, rep)
    rng = np.random.default_rng(0)
    off = g["offsets"].numpy()
    if name in FULL_EVERY_ROW:
        H.check_ffn(w, inp, g, n, rep)
        H.check_combine(w, g, rep)
        H.check_end_to_end(w, inp, g, idx, gates, rep)
    else:
        rows = sampled_rows(off, rng)
        H.check_ffn(w, inp, g, n, rep, rows=rows)
        rep["ffn_rows_checked"] = len(rows)
        toks = sorted(set(rng.choice(w.T, size=min(w.T, 512), replace=False).tolist())
                      | {0, w.T - 1})
        H.check_combine(w, g, rep, rows=toks)
        H.check_end_to_end(w, inp, g, idx, gates, rep, rows=toks)
    H.check_gather_path(w, g, rep)
    f = H.run_forward(w, dev)
    assert f["device_error"] == 0
    assert torch.equal(f["y"], g["y"])
    print(name, rep)


def test_bf16_to_f16_reencoding():
    """The library's re-encoding equals a round-to-nearest-even conversion and is exact
    for every value of magnitude >= 2^-17 (the count of inexact values is reported)."""
    import sparsely_gated_mixture_moe_b200 as moe
    w2 = workloads.make_inputs(W["switch"].scaled(T=16))["w2"]
    special = torch.tensor([0.0, -0.0, 2.0 ** -17, 2.0 ** -18, 3.0 * 2.0 ** -20, 65504.0, 1e5,
                            -1e-30, 1.0 + 2.0 ** -7], dtype=torch.bfloat16)
    for src in (w2.reshape(-1), special):
        ref = src.to(torch.float16)
        inexact_cpu = int((ref.double() != src.double()).sum())
        dst = torch.empty(src.shape, dtype=torch.float16, device="cuda")
        cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
        moe.moe_bf16_to_f16(src.cuda(), dst, n_inexact=cnt)
        assert torch.equal(dst.cpu().view(torch.int16), ref.view(torch.int16))
        assert int(cnt.item()) == inexact_cpu
        big = src.double().abs() >= 2.0 ** -17
        fin = src.double().abs() <= 65504
        assert torch.equal(ref.double()[big & fin], src.double()[big & fin])


def test_fast_erf_matches_cuda_erff():
    """The GELU epilogue's erf (Abramowitz & Stegun 7.1.26) stays within 1e-6 of CUDA's
    erff: the formula's 1.5e-7 plus its fp32 evaluation with the fast reciprocal and
    exponential (a few ulp of 1 each).  The activations it feeds are rounded to fp16 or
    bf16 (half-ulp >= 2.4e-4 relative), so this is three orders of magnitude below."""
    import ctypes
    import sparsely_gated_mixture_moe_b200 as moe
    x = torch.cat([torch.linspace(-12, 12, 2_000_001), torch.tensor(
        [0.0, -0.0, 1e-30, -1e-30, float("inf"), float("-inf"), 3.4e38, -3.4e38])]).cuda()
    fast, ref = torch.empty_like(x), torch.empty_like(x)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    assert moe.lib.moe_erf_check(p(x), p(fast), p(ref), x.numel(), None) == 0
    torch.cuda.synchronize()
    d = (fast - ref).abs()
    assert float(d.max()) <= 1e-6, float(d.max())
    assert fast[-4].item() == 1.0 and fast[-3].item() == -1.0


def test_packed_gelu_matches_exact_gelu():
    """The up-projection's GELU epilogue (A&S 7.1.26 erf evaluated on f32x2 pairs) stays
    within 2e-7 |z| + 1e-6 of 0.5 z (1 + erff(z / sqrt 2)): the formula's 1.5e-7 on erf,
    scaled by z / 2, plus a few fp32 roundings.  Its results are rounded to 16 bits
    (half-ulp >= 2.4e-4 relative) before anything else reads them."""
    import ctypes
    import sparsely_gated_mixture_moe_b200 as moe
    z = torch.cat([torch.linspace(-12, 12, 2_000_001), torch.tensor(
        [0.0, -0.0, 1e-30, -1e-30, 3.0e4, -3.0e4, 1e-3])]).cuda()  # odd count: last pairs with itself
    fast, ref = torch.empty_like(z), torch.empty_like(z)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    assert moe.lib.moe_gelu_check(p(z), p(fast), p(ref), z.numel(), None) == 0
    torch.cuda.synchronize()
    bound = 2e-7 * z.abs() + 1e-6
    d = (fast - ref).abs()
    assert bool((d <= bound).all()), float((d - bound).max())
    assert fast[-3].item() == 3.0e4 and fast[-2].item() == 0.0
    assert moe.lib.moe_gelu_check(p(z), p(fast), p(ref), -1, None) != 0


@pytest.mark.parametrize("name,launches", [("switch", 1), ("three_kernel_permute_T200k", 3)])
def test_permute_launch_path(name, launches):
    """moe_permute runs as one launch (grid barriers between its phases) when every block
    of that grid fits on the GPU at once, and as three kernels otherwise."""
    import sparsely_gated_mixture_moe_b200 as moe
    w = FULL[name]
    cfg = H.config_of(w)
    dev = H.to_device(workloads.make_inputs(w))
    n = w.T * w.k
    gen = torch.Generator().manual_seed(7)
    idx = torch.randint(0, w.E, (w.T, w.k), generator=gen, dtype=torch.int32).cuda()
    o = {key: torch.empty(size, dtype=torch.int32, device="cuda")
         for key, size in (("counts", w.E), ("offsets", w.E + 1), ("perm_src", n), ("slot_pos", n))}
    x_perm = torch.empty(n, w.d_model, dtype=w.torch_dtype, device="cuda")
    ws = moe.workspace(cfg)
    moe.moe_permute(cfg, idx, dev["x"], o["counts"], o["offsets"], o["perm_src"], o["slot_pos"],
                    x_perm, ws)
    assert moe.last_launch_count() == launches
    assert moe.moe_get_error(ws) == 0
    assert o["counts"].tolist() == torch.bincount(idx.view(-1).long(), minlength=w.E).tolist()
    # index arrays only: the three-kernel path leaves out its row-copy kernel
    moe.moe_permute(cfg, idx, None, o["counts"], o["offsets"], o["perm_src"], o["slot_pos"],
                    None, ws)
    assert moe.last_launch_count() == min(launches, 2)
    assert moe.moe_get_error(ws) == 0


Y_BF16 = {
    # k = 2 through the combine kernel, several tiles with a ragged tail
    "combine_k2": Workload("yk2", T=1000, d_model=256, d_ff=512, E=8, k=2, act="gelu"),
    # k = 1 through the fused down-projection epilogue, with dropped tokens (zero rows)
    "fused_k1_drops": Workload("yk1", T=1500, d_model=256, d_ff=512, E=8, k=1, renorm=False,
                               capacity_factor=0.9, act="gelu"),
    "noisy_k4": W["noisy"].scaled(T=700),
    "zipf_full": W["zipf"],
    "switch_full": W["switch"],
}


@pytest.mark.parametrize("name", list(Y_BF16))
def test_bf16_output_is_the_rounded_fp32_output(name):
    """With y_bf16 the layer output is the fp32 output rounded once to bf16 (nearest even),
    bit for bit: on the combine kernel (k >= 2) and on the fused down-projection epilogue
    (k = 1), whose dropped tokens' rows are zero.  So it inherits the fp32 output's parity
    with the oracle, plus one bf16 rounding (<= 2^-9 relative)."""
    import sparsely_gated_mixture_moe_b200 as moe
    w = Y_BF16[name]
    dev = H.to_device(workloads.make_inputs(w))
    weights = {kk: v for kk, v in dev.items() if kk not in ("x", "noise")}
    cfg32 = H.config_of(w)
    cfg16 = H.config_of(w)
    cfg16.y_bf16 = 1
    l32 = moe.MoELayer(cfg32, weights)
    y32 = l32.forward(dev["x"], noise=dev.get("noise")).clone()
    del l32
    l16 = moe.MoELayer(cfg16, weights)
    y16 = l16.forward(dev["x"], noise=dev.get("noise"))
    torch.cuda.synchronize()
    assert y16.dtype == torch.bfloat16
    assert moe.moe_get_error(l16.ws) == 0
    assert torch.equal(y16, y32.to(torch.bfloat16))
    if name == "fused_k1_drops":  # some expert overflows its capacity: zero rows exist
        assert int(l16.counts.max()) > moe.moe_capacity(cfg16)
        assert bool((y16.float().abs().sum(1) == 0).any())


FUSED_K2 = {
    # y (32 MB) in 2048 zeroing chunks against ~256 up-projection pair tiles: most chunks
    # are zeroed after a CTA's last tile
    "zero_tail_T8192": Workload("fk2", T=8192, d_model=1024, d_ff=1024, E=8, k=2, act="gelu"),
    # capacity drops: tokens with one or no kept assignment (rows that only the zeroing
    # writes), 128-row tiles
    "drops_T6000": Workload("fk2c", T=6000, d_model=512, d_ff=512, E=32, k=2, act="relu",
                            capacity_factor=0.6),
    "zipf_full": W["zipf"],
}


@pytest.mark.parametrize("name", list(FUSED_K2))
def test_fused_top2_combine_covers_every_row(name):
    """moe_expert_ffn_combine with k = 2 into a y filled with NaN: the up-projection must
    zero every row and the down-projection add each kept row into its token, so y is
    finite everywhere, zero exactly for the tokens with no kept assignment, within one
    rounding of the second product of moe_expert_ffn + moe_combine, and the same bits on
    a second run (the two in-memory adds of a token commute)."""
    import sparsely_gated_mixture_moe_b200 as moe
    w = FUSED_K2[name]
    dev = H.to_device(workloads.make_inputs(w))
    cfg = H.config_of(w)
    assert moe.fused_combine(cfg)
    T, k, E, d, f = w.T, w.k, w.E, w.d_model, w.d_ff
    cu = "cuda"
    o = {"idx": torch.empty(T, k, dtype=torch.int32, device=cu),
         "gate": torch.empty(T, k, device=cu),
         "counts": torch.empty(E, dtype=torch.int32, device=cu),
         "offsets": torch.empty(E + 1, dtype=torch.int32, device=cu),
         "perm_src": torch.empty(T * k, dtype=torch.int32, device=cu),
         "slot_pos": torch.empty(T * k, dtype=torch.int32, device=cu),
         "x_perm": torch.empty(T * k, d, dtype=torch.bfloat16, device=cu),
         "h": torch.empty(T * k, f, dtype=torch.bfloat16, device=cu),
         "y_perm": torch.empty(T * k, d, device=cu), "y": torch.empty(T, d, device=cu)}
    ws = moe.workspace(cfg)
    moe.moe_route(cfg, dev["x"], dev["w_gate"], o["idx"], o["gate"], ws,
                  logit_bias=dev.get("logit_bias"))
    moe.moe_permute(cfg, o["idx"], dev["x"], o["counts"], o["offsets"], o["perm_src"],
                    o["slot_pos"], o["x_perm"], ws)
    moe.moe_expert_ffn(cfg, o["x_perm"], o["offsets"], dev["w1"], dev["w2"], o["h"], o["y_perm"], ws)
    moe.moe_combine(cfg, o["y_perm"], o["slot_pos"], o["gate"], o["y"], ws)
    ys = []
    for _ in range(2):
        yf = torch.full((T, d), float("nan"), device=cu)
        moe.moe_expert_ffn_combine(cfg, o["x_perm"], o["offsets"], o["perm_src"], o["slot_pos"],
                                   o["gate"], dev["w1"], dev["w2"], o["h"], yf, ws)
        assert moe.last_launch_count() == 2
        ys.append(yf)
    torch.cuda.synchronize()
    assert moe.moe_get_error(ws) == 0
    assert torch.equal(ys[0], ys[1])
    yf, yc = ys[0].double(), o["y"].double()
    assert bool(torch.isfinite(yf).all())
    sp = o["slot_pos"].long().view(T, k)
    kept = (sp >= 0)
    none_kept = ~kept.any(1)
    if w.capacity_factor is not None:
        assert bool(none_kept.any()) and bool((kept.sum(1) == 1).any())
    assert bool((yf[none_kept] == 0).all())
    yp = o["y_perm"].double()[sp.clamp(min=0)]
    mag = (o["gate"].double().abs().view(T, k, 1) * yp.abs() * kept.double().unsqueeze(-1)).sum(1)
    assert bool(((yf - yc).abs() <= 2.0 ** -22 * mag).all()), float((yf - yc).abs().max())


def test_forward_replays_from_a_cuda_graph():
    """moe_forward captured into a CUDA graph (its kernels and their programmatic launch
    edges) and replayed gives the eager result bit for bit, also after the input changes
    in place."""
    import sparsely_gated_mixture_moe_b200 as moe
    w = W["switch"].scaled(T=2048)
    cfg = H.config_of(w)
    dev = H.to_device(workloads.make_inputs(w))
    layer = moe.MoELayer(cfg, {kk: v for kk, v in dev.items() if kk not in ("x", "noise")})
    x = dev["x"].clone()
    y1 = layer.forward(x).clone()
    x2 = workloads.make_inputs(w.scaled(T=2048, seed=5))["x"].cuda()
    layer.forward(x2)
    y2 = layer.y.clone()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="thread_local"):
        layer.forward(x)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(layer.y, y1)
    x.copy_(x2)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(layer.y, y2)
    assert moe.moe_get_error(layer.ws) == 0


def test_bounded_wait_expires_and_reports_timeout():
    """A grid barrier that can never complete (failure detection without a fault): each
    block's wait gives up after its limit, the timeout bit reaches the host through the
    error word, and the same workspace then serves a normal permutation exactly (the
    barrier counters were reset and the context is still usable)."""
    import ctypes
    import sparsely_gated_mixture_moe_b200 as moe
    from oracle import moe_oracle as orc
    w = W["switch"].scaled(T=4096)
    cfg = H.config_of(w)
    ws = moe.workspace(cfg)
    assert moe.lib.moe_wait_timeout_check(ctypes.c_void_p(ws.data_ptr()), None) == 0
    assert moe.moe_get_error(ws) == 8          # MOE_DEVERR_TIMEOUT, and cleared
    assert moe.moe_get_error(ws) == 0
    dev = H.to_device(workloads.make_inputs(w))
    gen = torch.Generator().manual_seed(3)
    idx = torch.randint(0, w.E, (w.T, w.k), generator=gen, dtype=torch.int32)
    n = w.T * w.k
    o = {key: torch.empty(size, dtype=torch.int32, device="cuda")
         for key, size in (("counts", w.E), ("offsets", w.E + 1), ("perm_src", n), ("slot_pos", n))}
    x_perm = torch.empty(n, w.d_model, dtype=w.torch_dtype, device="cuda")
    moe.moe_permute(cfg, idx.cuda(), dev["x"], o["counts"], o["offsets"], o["perm_src"],
                    o["slot_pos"], x_perm, ws)
    assert moe.last_launch_count() == 1
    assert moe.moe_get_error(ws) == 0
    C = orc.capacity(w.capacity_factor, w.T, w.k, w.E)
    counts, offsets, perm_src, slot_pos = orc.dispatch(idx.long().numpy(), w.E, C)
    assert o["counts"].cpu().tolist() == counts.tolist()
    assert o["offsets"].cpu().tolist() == offsets.tolist()
    kept = int(offsets[-1])
    assert o["perm_src"][:kept].cpu().tolist() == perm_src.tolist()
    assert o["slot_pos"].cpu().tolist() == slot_pos.tolist()
