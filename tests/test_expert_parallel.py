"""Expert parallelism's exchange, on CPU with two gloo ranks (no GPU).

Each rank routes its own batch with the oracle, sends its kept rows with the library's
exchange helpers (`exchange_plan`, `dispatch_rows`, `return_rows`: one message per
(rank, expert) run, landing expert-major), runs the experts it holds on the rows it
received with the oracle's expert function (one group per local expert, as
ExpertParallelMoE hands them to moe_expert_ffn_grouped), sends the outputs back and
combines them.  The result must equal the oracle's
single-device layer on the same rank's batch: every row reached the right expert and
came back to the right slot.  The compute here is the oracle's; the kernels' side of the
same grouping is tested on the GPU (tests/test_gpu_expert_parallel.py)."""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads
from oracle import moe_oracle as orc
from sparsely_gated_mixture_moe_b200 import expert_parallel as ep
from workloads import Workload

CASES = {
    "k2_no_capacity": Workload("ep2", T=96, d_model=32, d_ff=64, E=4, k=2, act="gelu"),
    "k1_capacity_drops": Workload("ep1", T=120, d_model=32, d_ff=48, E=8, k=1, renorm=False,
                                  capacity_factor=0.75, act="relu"),
    "k4_noisy": Workload("ep4", T=64, d_model=32, d_ff=32, E=8, k=4, gating="noisy_topk",
                         act="relu"),
}


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_inputs(w, rank):
    """Shared weights (the workload's seed) and this rank's own tokens (and noise)."""
    shared = workloads.make_inputs(w)
    own = workloads.make_inputs(w.scaled(seed=rank + 1))
    inp = dict(shared)
    inp["x"] = own["x"]
    if "noise" in own:
        inp["noise"] = own["noise"]
    return inp


def _worker(rank, world, port, name, q):
    try:
        dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank,
                                world_size=world)
        w = CASES[name]
        inp = _rank_inputs(w, rank)
        T, k, E = w.T, w.k, w.E
        e0, e1 = ep.local_expert_range(E, world, rank)
        El = e1 - e0
        r = orc.route(inp, w)
        C = orc.capacity(w.capacity_factor, T, k, E)   # per rank: its batch is one group
        counts, offsets, perm_src, slot_pos = orc.dispatch(r["idx"], E, C)
        x_perm = torch.from_numpy(orc.gather_rows(inp["x"], perm_src, k))
        kept = torch.from_numpy(np.diff(offsets))
        plan = ep.exchange_plan(kept, world)
        # what every rank sends to every other, gathered, so the plan can be checked
        all_kept = [torch.zeros_like(kept) for _ in range(world)]
        dist.all_gather(all_kept, kept)
        want_recv = [[int(v) for v in a.reshape(world, El)[rank]] for a in all_kept]
        assert plan.recv_counts == want_recv
        assert plan.send_counts == [[int(v) for v in row] for row in kept.reshape(world, El)]
        recv_buf = torch.zeros(world * T * k, w.d_model, dtype=torch.float64)
        recv = ep.dispatch_rows(x_perm, plan, recv_buf)
        off = plan.expert_offsets.numpy()
        assert off[-1] == plan.rows_in == recv.shape[0]
        y_recv = torch.zeros(world * T * k, w.d_model, dtype=torch.float64)
        w1, w2 = inp["w1"], inp["w2"]
        for e in range(El):
            a, b = int(off[e]), int(off[e + 1])
            if b > a:
                y_recv[a:b] = torch.from_numpy(orc.expert(recv[a:b].numpy(), w1[e0 + e], w2[e0 + e],
                                                          w.act)[1])
        back = torch.zeros(int(offsets[-1]), w.d_model, dtype=torch.float64)
        ep.return_rows(y_recv, plan, back)
        y = orc.combine(back.numpy(), slot_pos, r["gates"], T, k)
        ref = orc.moe_forward(inp, w)["y"]
        err = float(np.max(np.abs(y - ref)))
        q.put((rank, err, plan.rows_in, None))
        dist.barrier()
        dist.destroy_process_group()
    except Exception as exc:  # report to the parent instead of hanging it
        q.put((rank, None, None, repr(exc)))


@pytest.mark.parametrize("name", list(CASES))
def test_expert_parallel_exchange_two_ranks(name):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, name, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    for rank, err, rows_in, exc in results:
        assert exc is None, (rank, exc)
        assert err <= 1e-12, (rank, err)
        assert rows_in > 0


def test_local_expert_range_and_plan_single_rank():
    assert ep.local_expert_range(8, 2, 0) == (0, 4) and ep.local_expert_range(8, 2, 1) == (4, 8)
    with pytest.raises(ValueError):
        ep.local_expert_range(6, 4, 0)
    kept = torch.tensor([3, 0, 5, 2])
    plan = ep.exchange_plan(kept, 1)
    assert plan.send_counts == [[3, 0, 5, 2]] and plan.recv_counts == [[3, 0, 5, 2]]
    assert plan.send_pos == [[0, 3, 3, 8]] and plan.recv_pos == [[0, 3, 3, 8]]
    assert plan.expert_offsets.tolist() == [0, 3, 3, 8, 10]
    rows = torch.arange(10.0).reshape(10, 1)
    out = torch.zeros(10, 1)
    assert torch.equal(ep.dispatch_rows(rows, plan, out), rows)
