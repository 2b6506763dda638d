"""The expert-parallel layer's kernels on one GPU.

moe_expert_ffn_grouped runs the rows an expert-parallel rank receives: R sources, each
sending rows for the E_local experts this rank holds, laid out source by source and,
within a source, expert by expert (group g = s * E_local + e uses weights g mod
E_local).  Each output row depends only on its own input row and its expert's weights,
and the tensor-core accumulation order over K does not depend on which other rows share
the tile, so the grouped result must equal, row for row and bit for bit, moe_expert_ffn
on the same rows regrouped expert by expert; sampled rows are also checked against the
fp64 oracle.  ExpertParallelMoE on a single rank (no exchange) must give MoELayer's
output bit for bit, and so must each of two ranks run as two processes on this GPU,
each holding half of the experts, exchanging their runs of rows through gloo (staged
through host memory; every wait is on the host, no kernel waits for another process).
The exchange alone is also tested on CPU (tests/test_expert_parallel.py)."""
import numpy as np
import pytest
import torch

import workloads
from oracle import moe_oracle as orc
from tests import gpu_harness as H
from workloads import Workload

pytestmark = pytest.mark.gpu

GROUPED = {
    # (sources R, local experts, d, f, max rows per (source, expert), act, seed)
    "R3_E4_single_cta_tiles": (3, 4, 256, 512, 300, "gelu", 0),
    "R2_E2_pair_tiles": (2, 2, 256, 512, 1400, "relu", 1),
    "R4_E1_one_expert": (4, 1, 128, 256, 500, "gelu", 2),
}


def _weights(E, d, f, seed):
    g = torch.Generator().manual_seed(1000 + seed)
    w1 = (torch.randn(E, f, d, generator=g) * d ** -0.5).to(torch.bfloat16)
    w2 = (torch.randn(E, d, f, generator=g) * f ** -0.5).to(torch.bfloat16)
    return w1, w2


@pytest.mark.parametrize("name", list(GROUPED))
def test_grouped_ffn_equals_expert_ffn_row_for_row(name):
    import sparsely_gated_mixture_moe_b200 as moe
    R, El, d, f, most, act, seed = GROUPED[name]
    g = torch.Generator().manual_seed(seed)
    counts = torch.randint(0, most + 1, (R, El), generator=g)
    counts[0, 0] = 0  # an empty group
    rows = int(counts.sum())
    x = torch.randn(rows, d, generator=g).to(torch.bfloat16)
    w1, w2 = _weights(El, d, f, seed)
    off_g = np.zeros(R * El + 1, np.int64)
    off_g[1:] = np.cumsum(counts.reshape(-1).numpy())
    # the same rows regrouped expert by expert (sources in order within an expert)
    order = []
    for e in range(El):
        for s in range(R):
            gi = s * El + e
            order.extend(range(int(off_g[gi]), int(off_g[gi + 1])))
    order = np.asarray(order, np.int64)
    off_e = np.zeros(El + 1, np.int64)
    off_e[1:] = np.cumsum(counts.sum(0).numpy())

    cfg = moe.make_config(rows, d, f, El, 1, act=act, dtype="bf16")
    cu = "cuda"
    xg = x.to(cu)
    h_g = torch.empty(rows, f, dtype=torch.bfloat16, device=cu)
    y_g = torch.full((rows, d), float("nan"), device=cu)
    ws = moe.workspace(cfg)
    moe.moe_expert_ffn_grouped(cfg, xg, torch.from_numpy(off_g).to(torch.int32).to(cu), R * El,
                               w1.to(cu), w2.to(cu), h_g, y_g, ws)
    assert moe.moe_get_error(ws) == 0
    xe = x[torch.from_numpy(order)].to(cu)
    h_e = torch.empty(rows, f, dtype=torch.bfloat16, device=cu)
    y_e = torch.empty(rows, d, device=cu)
    moe.moe_expert_ffn(cfg, xe, torch.from_numpy(off_e).to(torch.int32).to(cu), w1.to(cu),
                       w2.to(cu), h_e, y_e, ws)
    assert moe.moe_get_error(ws) == 0
    inv = torch.from_numpy(order).to(cu)
    assert torch.equal(y_g[inv], y_e)
    assert torch.equal(h_g[inv], h_e)
    # sampled rows against the fp64 oracle: each group's first and last row
    yc = y_g.cpu().double().numpy()
    worst = 0.0
    for gi in range(R * El):
        a, b = int(off_g[gi]), int(off_g[gi + 1])
        if b <= a:
            continue
        e = gi % El
        for rr in sorted({a, b - 1}):
            _, yo = orc.expert(x[rr:rr + 1].float().numpy(), w1[e], w2[e], act)
            worst = max(worst, float(np.max(np.abs(yc[rr] - yo[0])) / (np.sqrt(np.mean(yo ** 2)) + 1e-30)))
    assert worst <= 2e-2, worst


def test_grouped_ffn_validates_and_reports_bad_offsets():
    import ctypes
    import sparsely_gated_mixture_moe_b200 as moe
    cfg = moe.make_config(64, 128, 128, 2, 1, dtype="bf16")
    cu = "cuda"
    x = torch.zeros(64, 128, dtype=torch.bfloat16, device=cu)
    w1 = torch.zeros(2, 128, 128, dtype=torch.bfloat16, device=cu)
    w2 = torch.zeros(2, 128, 128, dtype=torch.bfloat16, device=cu)
    h = torch.empty(64, 128, dtype=torch.bfloat16, device=cu)
    y = torch.empty(64, 128, device=cu)
    ws = moe.workspace(cfg)
    bad = torch.tensor([0, 40, 20, 64, 64], dtype=torch.int32, device=cu)  # decreasing
    moe.moe_expert_ffn_grouped(cfg, x, bad, 4, w1, w2, h, y, ws)
    err = moe.moe_get_error(ws)
    assert err & moe.DEVERR["offsets"]
    c32 = moe.make_config(64, 128, 128, 2, 1, dtype="f32")
    P = ctypes.c_void_p(x.data_ptr())
    assert moe.lib.moe_expert_ffn_grouped(ctypes.byref(c32), P, 64, P, 4, P, P, P, P, P, None) == 2
    assert moe.lib.moe_expert_ffn_grouped(ctypes.byref(cfg), P, 64, P, 0, P, P, P, P, P, None) == 1


EP_SINGLE = {
    "k2_gelu": Workload("eps2", T=1500, d_model=256, d_ff=512, E=8, k=2, act="gelu"),
    "k1_capacity": Workload("eps1", T=2048, d_model=256, d_ff=512, E=16, k=1, renorm=False,
                            capacity_factor=1.0, act="gelu"),
    "noisy_k4": workloads.WORKLOADS["noisy"].scaled(T=900),
}


@pytest.mark.parametrize("name", list(EP_SINGLE))
def test_expert_parallel_single_rank_equals_layer(name):
    import sparsely_gated_mixture_moe_b200 as moe
    from sparsely_gated_mixture_moe_b200.expert_parallel import ExpertParallelMoE
    w = EP_SINGLE[name]
    dev = H.to_device(workloads.make_inputs(w))
    weights = {kk: v for kk, v in dev.items() if kk not in ("x", "noise")}
    cfg = H.config_of(w)
    layer = moe.MoELayer(cfg, weights)
    y_ref = layer.forward(dev["x"], noise=dev.get("noise")).clone()
    epl = ExpertParallelMoE(H.config_of(w), weights)
    y = epl.forward(dev["x"], noise=dev.get("noise"))
    torch.cuda.synchronize()
    assert moe.moe_get_error(epl.ws) == 0
    assert epl.world == 1 and epl.plan.rows_in == epl.plan.rows_out
    assert torch.equal(y, y_ref)


EP_TWO_RANKS = {
    "k2_gelu": Workload("ept2", T=1200, d_model=256, d_ff=512, E=8, k=2, act="gelu"),
    "k1_capacity": Workload("ept1", T=1600, d_model=256, d_ff=512, E=16, k=1, renorm=False,
                            capacity_factor=1.0, act="gelu"),
    "noisy_k4": workloads.WORKLOADS["noisy"].scaled(T=700),
}


def _ep_rank(rank, world, port, name, q):
    try:
        import torch.distributed as dist
        import sparsely_gated_mixture_moe_b200 as moe
        from sparsely_gated_mixture_moe_b200.expert_parallel import (ExpertParallelMoE,
                                                                     local_expert_range)
        from tests.test_expert_parallel import _rank_inputs
        torch.cuda.set_device(0)
        dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank,
                                world_size=world)
        w = EP_TWO_RANKS[name]
        dev = H.to_device(_rank_inputs(w, rank))
        full = {kk: v for kk, v in dev.items() if kk not in ("x", "noise")}
        e0, e1 = local_expert_range(w.E, world, rank)
        mine = dict(full, w1=full["w1"][e0:e1].contiguous(), w2=full["w2"][e0:e1].contiguous())
        epl = ExpertParallelMoE(H.config_of(w), mine)
        y = epl.forward(dev["x"], noise=dev.get("noise")).clone()
        err = moe.moe_get_error(epl.ws)
        layer = moe.MoELayer(H.config_of(w), full)
        y_ref = layer.forward(dev["x"], noise=dev.get("noise"))
        torch.cuda.synchronize()
        sent_away = sum(sum(r) for i, r in enumerate(epl.plan.send_counts) if i != rank)
        q.put((rank, err, bool(torch.equal(y, y_ref)), sent_away, None))
        dist.barrier()
        dist.destroy_process_group()
    except Exception as exc:  # report to the parent instead of hanging it
        q.put((rank, None, None, None, repr(exc)))


@pytest.mark.parametrize("name", list(EP_TWO_RANKS))
def test_expert_parallel_two_ranks_on_one_gpu(name):
    import torch.multiprocessing as mp
    from tests.test_expert_parallel import _free_port
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_rank, args=(r, world, port, name, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    for rank, err, equal, sent_away, exc in results:
        assert exc is None, (rank, exc)
        assert err == 0, (rank, err)
        assert sent_away > 0, rank   # rows really crossed to the other rank
        assert equal, rank
