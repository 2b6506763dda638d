"""Host-side logic of bench.py without a GPU: the max-over-ranks reduction on a real
2-rank gloo process group, the clock-sample parser, the algorithmic byte/FLOP counts and
the reference arm's JSON line."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        assert bench.dist_env() == (rank, rank, world)
        v = bench.max_over_ranks(1.5 + 10.0 * rank)
        out.put((rank, v))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert got == [(0, 11.5), (1, 11.5)]


def test_max_over_ranks_single_process_is_identity():
    assert bench.max_over_ranks(3.25) == 3.25


def test_clock_summary_parser():
    c = bench.ClockSampler(0)
    c.lines = [
        "0, 1965, 1965, 300.5, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1830, 1965, 990.1, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1800, 1965, 995.0, 0x4, Not Active, Not Active, Not Active, Active",
        "garbage line",
    ]
    s = c.summary()
    assert s["sm_max_mhz"] == 1965 and s["samples"] == 3
    assert s["sm_mhz"] == 1830
    assert s["reasons"] == ["sw_power_cap"]


def test_algorithmic_counts_switch():
    w = workloads.WORKLOADS["switch"]
    kept = [128] * 128
    a = bench.algorithmic(w, 16384, kept)
    assert a["ffn_flops"] == 4.0 * 16384 * 768 * 3072
    weights = 128 * 2 * 768 * 3072 * 2
    assert a["ffn_bytes"] == weights + 16384 * 768 * 2 + 16384 * 768 * 4
    assert a["permute_bytes"] == 16384 * 12 + 128 * 8 + 16384 * 768 * 2 * 2
    assert a["route_bytes"] == 16384 * 768 * 2 + 128 * 768 * 2 + 16384 * 8
    # y is fp32 in the benchmark figures (4 bytes per value written) unless --y-bf16
    assert not bench.y_bf16_of(w)
    assert a["combine_bytes"] == 16384 * 768 * 4 + 16384 * 8 + 16384 * 768 * 4
    f = bench.algorithmic(w, 16384, kept, fused=True)
    assert f["combine_bytes"] == 0.0
    assert f["ffn_bytes"] == weights + 16384 * 768 * 2 + 16384 * 768 * 4 + 16384 * 8 + 16384 * 4
    # k = 2 fused: y zeroed (written once) and every kept row added into it
    z = workloads.WORKLOADS["zipf"]
    zk = [8192] * 16
    fz = bench.algorithmic(z, 131072, zk, fused=True)
    assert fz["combine_bytes"] == 0.0
    assert fz["ffn_bytes"] == (16 * 2 * 1024 * 4096 * 2 + 131072 * 1024 * 2 + 65536 * 1024 * 4
                               + 131072 * 8 + 131072 * 1024 * 4)
    bench.Y_BF16 = True
    try:
        assert bench.y_bf16_of(w) and not bench.y_bf16_of(workloads.WORKLOADS["tiny"])
        b16 = bench.algorithmic(w, 16384, kept)
        assert b16["combine_bytes"] == 16384 * 768 * 4 + 16384 * 8 + 16384 * 768 * 2
    finally:
        bench.Y_BF16 = False


def test_reference_arm_json_line():
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "3"])
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s"
    assert line["metric"] == bench.METRIC and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["T"] == 512
