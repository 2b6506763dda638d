"""moe_permute_noalloc: the permutation step for callers that cannot allocate device
memory (a host runtime that owns every device buffer, a latency path that cannot afford
cudaMalloc's synchronisation, a callback where allocation is not allowed).  It keeps its
scratch in a fixed array inside the library, so it takes no workspace.

The test calls it through the C ABI twice in a row on the same inputs and checks both
results against moe_permute (the workspace version) bit for bit -- the permutation is
integer and byte work, where the parity bar is exactness.  It must pass run alone in a
fresh process and after the other tests (the fixed array keeps the previous call's
contents, which the entry point must not depend on).  This file is named so that pytest
collects it last."""
import ctypes

import pytest
import torch

import sparsely_gated_mixture_moe_b200 as moe
import workloads
from workloads import Workload

pytestmark = pytest.mark.gpu

CASES = {
    "switch_T2048": workloads.WORKLOADS["switch"].scaled(T=2048),
    "zipf_T4096": workloads.WORKLOADS["zipf"].scaled(T=4096),
    "noisy_T1024": workloads.WORKLOADS["noisy"].scaled(T=1024),
    "cap0.25_f32": Workload("c", T=777, d_model=64, d_ff=64, E=8, k=2, capacity_factor=0.25,
                            dtype="f32"),
}


def _cfg(w):
    return moe.make_config(w.T, w.d_model, w.d_ff, w.E, w.k, gating=w.gating, renorm=w.renorm,
                           capacity_factor=w.capacity_factor, act=w.act, dtype=w.dtype)


def _outputs(w):
    n = w.T * w.k
    return {"counts": torch.full((w.E,), -5, dtype=torch.int32, device="cuda"),
            "offsets": torch.full((w.E + 1,), -5, dtype=torch.int32, device="cuda"),
            "perm_src": torch.full((n,), -5, dtype=torch.int32, device="cuda"),
            "slot_pos": torch.full((n,), -5, dtype=torch.int32, device="cuda"),
            "x_perm": torch.zeros(n, w.d_model, dtype=w.torch_dtype, device="cuda")}


def _noalloc(cfg, idx, x, o):
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = moe.lib.moe_permute_noalloc(ctypes.byref(cfg), p(idx), p(x), p(o["counts"]),
                                     p(o["offsets"]), p(o["perm_src"]), p(o["slot_pos"]),
                                     p(o["x_perm"]), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, moe.lib.moe_status_string(st)


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_permute_matches_workspace_permute(name):
    w = CASES[name]
    cfg = _cfg(w)
    inp = {k: v.cuda() for k, v in workloads.make_inputs(w).items()}
    # expert choices from the router, then the workspace version as the reference
    idx = torch.empty(w.T, w.k, dtype=torch.int32, device="cuda")
    gate = torch.empty(w.T, w.k, dtype=torch.float32, device="cuda")
    ws = moe.workspace(cfg)
    moe.moe_route(cfg, inp["x"], inp["w_gate"], idx, gate, ws, w_noise=inp.get("w_noise"),
                  noise=inp.get("noise"), logit_bias=inp.get("logit_bias"))
    ref = _outputs(w)
    moe.moe_permute(cfg, idx, inp["x"], ref["counts"], ref["offsets"], ref["perm_src"],
                    ref["slot_pos"], ref["x_perm"], ws)
    assert moe.moe_get_error(ws) == 0
    n_kept = int(ref["offsets"][-1].item())
    for _ in range(2):
        got = _outputs(w)
        _noalloc(cfg, idx, inp["x"], got)
        torch.cuda.synchronize()
        for key in ("counts", "offsets", "slot_pos"):
            assert torch.equal(got[key], ref[key]), key
        assert torch.equal(got["perm_src"][:n_kept], ref["perm_src"][:n_kept])
        assert torch.equal(got["x_perm"][:n_kept], ref["x_perm"][:n_kept])


def _random_choices(T, k, E, seed):
    gen = torch.Generator().manual_seed(seed)
    return torch.randint(0, E, (T, k), generator=gen, dtype=torch.int32)


def test_noalloc_size_limit_boundary():
    """The scratch holds 256 bytes of counters and one int32 per (256-assignment chunk,
    expert): with E = 128 and k = 1 that allows T = 524,032 (2047 chunks) and refuses
    T = 524,033 (2048 chunks, 256 + 2048 * 512 bytes > 1 MiB) on the host, queueing
    nothing.  The largest accepted size runs and equals moe_permute bit for bit."""
    E, d = 128, 64
    too_big = moe.make_config(524_033, d, 64, E, 1)
    z = torch.zeros(16, dtype=torch.int32, device="cuda")
    p = ctypes.c_void_p(z.data_ptr())
    assert moe.lib.moe_permute_noalloc(ctypes.byref(too_big), p, p, p, p, p, p, p, None) == 2

    w = Workload("lim", T=524_032, d_model=d, d_ff=64, E=E, k=1)
    cfg = _cfg(w)
    x = workloads.make_x(w).cuda()
    idx = _random_choices(w.T, 1, E, 11).cuda()
    ref, got = _outputs(w), _outputs(w)
    ws = moe.workspace(cfg)
    moe.moe_permute(cfg, idx, x, ref["counts"], ref["offsets"], ref["perm_src"], ref["slot_pos"],
                    ref["x_perm"], ws)
    assert moe.moe_get_error(ws) == 0
    _noalloc(cfg, idx, x, got)
    torch.cuda.synchronize()
    for key in ("counts", "offsets", "perm_src", "slot_pos", "x_perm"):
        assert torch.equal(got[key], ref[key]), key


def test_noalloc_out_of_range_expert_is_dropped():
    """Without a device error word, an expert index outside [0, E) is dropped silently:
    its slot is -1, and counts and offsets tally only the valid entries."""
    w = Workload("oor", T=300, d_model=64, d_ff=64, E=8, k=2, dtype="f32")
    cfg = _cfg(w)
    x = workloads.make_x(w).cuda()
    idx = _random_choices(w.T, w.k, w.E, 5)
    bad = [(3, 0, -1), (10, 1, 8), (77, 0, 8), (299, 1, -1), (150, 0, 1000)]
    for t, j, v in bad:
        idx[t, j] = v
    got = _outputs(w)
    _noalloc(cfg, idx.cuda(), x, got)
    torch.cuda.synchronize()
    flat = idx.view(-1)
    valid = (flat >= 0) & (flat < w.E)
    tally = torch.bincount(flat[valid].long(), minlength=w.E)
    assert got["counts"].cpu().tolist() == tally.tolist()
    assert got["offsets"].cpu().tolist() == [0] + torch.cumsum(tally, 0).tolist()
    sp = got["slot_pos"].cpu()
    for t, j, _ in bad:
        assert int(sp[t * w.k + j]) == -1
    assert bool((sp[valid] >= 0).all())
