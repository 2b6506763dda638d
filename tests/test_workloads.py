"""The seeded input generator: determinism, shapes, dtypes, distributions and the
stored Zipf calibration (checked against the oracle's routing)."""
import json
import os

import numpy as np
import pytest
import torch

import workloads
from oracle import moe_oracle as orc


def test_five_workloads_shapes():
    W = workloads.WORKLOADS
    five = ["tiny", "switch", "noisy", "gshard", "zipf"]
    assert workloads.ORDER[:5] == five
    assert [W[n].T for n in five] == [512, 16384, 8192, 32768, 65536]
    assert [W[n].k for n in five] == [2, 1, 4, 2, 2]
    assert [W[n].E for n in five] == [8, 128, 256, 64, 16]
    h = W["hierarchical"]
    assert (h.groups, h.k_primary, h.E, h.k) == (8, 2, 128, 4)
    assert workloads.make_inputs(h.scaled(T=4, d_ff=64))["w_gate"].shape == (8 + 128, 512)
    assert orc.capacity(W["switch"].capacity_factor, 16384, 1, 128) == 160
    assert orc.capacity(W["gshard"].capacity_factor, 32768, 2, 64) == 2048


def test_inputs_deterministic_and_typed():
    w = workloads.WORKLOADS["noisy"].scaled(T=64, E=16, d_ff=128)
    a, b = workloads.make_inputs(w), workloads.make_inputs(w)
    for key in a:
        assert torch.equal(a[key], b[key])
    assert a["x"].dtype == torch.bfloat16 and a["noise"].dtype == torch.float32
    assert a["w1"].shape == (16, 128, 512) and a["w2"].shape == (16, 512, 128)
    assert a["w_gate"].shape == (16, 512) and a["w_noise"].shape == (16, 512)
    # independent streams: changing T leaves the weights untouched
    c = workloads.make_inputs(w.scaled(T=32))
    assert torch.equal(c["w1"], a["w1"]) and torch.equal(c["x"], a["x"][:32])


def test_distribution_scales():
    w = workloads.WORKLOADS["switch"].scaled(T=4096, E=4)
    inp = workloads.make_inputs(w)
    assert float(inp["x"].float().std()) == pytest.approx(1.0, rel=0.02)
    assert float(inp["w1"].float().std()) == pytest.approx(768 ** -0.5, rel=0.02)
    assert float(inp["w2"].float().std()) == pytest.approx(3072 ** -0.5, rel=0.02)


def test_zipf_calibration_reproduces():
    """The stored beta gives expert 0 a top-2 share within 0.5% of p_0 under the oracle's
    routing of the full skewed workload's tokens (a shorter prefix of tokens is used
    here to keep the CPU suite fast; the tolerance is widened accordingly)."""
    w = workloads.WORKLOADS["zipf"].scaled(T=8192)
    inp = workloads.make_inputs(w)
    idx = orc.top_k(orc.router_logits(inp["x"], inp["w_gate"], inp["logit_bias"]), w.k)
    share = float(np.sum(idx == 0)) / idx.size
    p0 = float(workloads.zipf_probs(16, 1.2)[0])
    assert share == pytest.approx(p0, rel=0.03)
    with open(os.path.join(os.path.dirname(workloads.__file__), "zipf_beta.json")) as f:
        meta = json.load(f)
    assert abs(meta["realised_share_expert0"] - p0) <= 0.005 * p0
