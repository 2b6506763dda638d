"""The C ABI without a GPU: the library loads, exports every function include/moe.h
declares, its config struct matches the header, host-side validation rejects bad
arguments before any CUDA call, and the capacity it computes equals the oracle's.

Every call here fails validation (or is a pure host query), so nothing is launched."""
import ctypes
import os
import re

import pytest

import sparsely_gated_mixture_moe_b200 as moe
from oracle import moe_oracle as orc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", src)))


def test_self_checks_validate_before_launching():
    """The erf and GELU self-check entry points refuse a negative count or a null
    pointer, and do nothing for n = 0 (no launch, so no GPU is needed here)."""
    for fn in (moe.lib.moe_erf_check, moe.lib.moe_gelu_check):
        assert fn(None, None, None, -1, None) == 1
        assert fn(None, None, None, 4, None) == 1
        assert fn(None, None, None, 0, None) == 0


def test_grouped_ffn_validates_before_launching():
    """moe_expert_ffn_grouped: fp32 layers are unsupported, groups must be positive and at
    most 1024, and zero rows launch nothing (no GPU needed for any of these)."""
    c = moe.make_config(64, 128, 128, 2, 1, dtype="bf16")
    c32 = moe.make_config(64, 128, 128, 2, 1, dtype="f32")
    f = moe.lib.moe_expert_ffn_grouped
    assert f(ctypes.byref(c32), FAKE, 64, FAKE, 4, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 2
    assert f(ctypes.byref(c), FAKE, 64, FAKE, 0, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert f(ctypes.byref(c), FAKE, 64, FAKE, 1025, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 2
    assert f(ctypes.byref(c), FAKE, -1, FAKE, 4, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert f(ctypes.byref(c), FAKE, 0, None, 4, None, None, None, None, None, None) == 0
    assert f(ctypes.byref(c), None, 64, FAKE, 4, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert f(ctypes.byref(c), FAKE_ODD, 64, FAKE, 4, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1


def test_library_exports_every_declared_symbol():
    names = _declared_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(moe.lib, n), n


def test_config_struct_layout():
    # int64 T, six int32, float, six int32 -> 60 bytes, 64 with 8-byte alignment
    assert ctypes.sizeof(moe.MoEConfig) == 64
    assert moe.MoEConfig.capacity_factor.offset == 32
    assert moe.MoEConfig.dtype.offset == 40
    assert moe.MoEConfig.hidden_f16.offset == 44
    assert moe.MoEConfig.groups.offset == 48
    assert moe.MoEConfig.k_primary.offset == 52
    assert moe.MoEConfig.y_bf16.offset == 56


def test_status_strings():
    for s in range(5):
        assert moe.lib.moe_status_string(s)


@pytest.mark.parametrize("cf,T,k,E", [(1.25, 16384, 1, 128), (2.0, 32768, 2, 64), (0.25, 100, 2, 8),
                                      (1.0, 10, 1, 4), (1.0, 8, 1, 4), (0.3, 10, 1, 4),
                                      (0.1, 1000, 2, 7), (1.1, 333, 3, 17), (3.7, 65536, 2, 16),
                                      (None, 10, 1, 4)])
def test_capacity_matches_oracle(cf, T, k, E):
    c = moe.make_config(T, 64, 64, E, k, capacity_factor=cf)
    want = orc.capacity(cf, T, k, E)
    assert moe.moe_capacity(c) == (-1 if want is None else want)


def _cfg(**kw):
    base = dict(T=256, d_model=128, d_ff=256, E=8, k=2, gating="softmax_topk", renorm=True,
                capacity_factor=None, act="relu", dtype="bf16")
    base.update(kw)
    return moe.make_config(**base)


FAKE = ctypes.c_void_p(0x100000)       # never dereferenced: every call below fails validation
FAKE_ODD = ctypes.c_void_p(0x100004)   # not 16-byte aligned


def _route(c, x=FAKE, wg=FAKE, wn=None, noise=None, idx=FAKE, gate=FAKE, load=None, ws=FAKE):
    return moe.lib.moe_route(ctypes.byref(c), x, wg, wn, noise, None, idx, gate, None, load, None,
                             ws, None)


def test_route_validation():
    assert _route(_cfg(), x=None) == 1
    assert _route(_cfg(), idx=None) == 1
    assert _route(_cfg(), ws=None) == 1
    assert _route(_cfg(), x=FAKE_ODD) == 1
    assert _route(_cfg(k=9, E=8)) == 1                      # k > E
    assert _route(_cfg(k=9, E=16)) == 2                     # k > 8 unsupported
    assert _route(_cfg(d_model=96)) == 2                    # bf16 needs d % 64
    assert _route(_cfg(d_model=100, dtype="f32")) == 2      # d % 8
    assert _route(_cfg(E=300, k=2)) == 2                    # bf16 E <= 256
    assert _route(_cfg(gating="noisy_topk")) == 1           # noisy without w_noise / noise
    assert _route(_cfg(), load=FAKE) == 1                   # load needs noisy gating
    assert _route(_cfg(gating="noisy_topk", E=4, k=4), wn=FAKE, noise=FAKE, load=FAKE) == 1
    bad = _cfg()
    bad.dtype = 7
    assert _route(bad) == 1
    bad = _cfg()
    bad.act = 5
    assert _route(bad) == 1
    assert _route(_cfg(y_bf16=True, dtype="f32")) == 1      # bf16 output of an fp32 layer
    bad = _cfg()
    bad.y_bf16 = 2
    assert _route(bad) == 1
    bad = _cfg()
    bad.T = -1
    assert _route(bad) == 1
    bad = _cfg()
    bad.hidden_f16 = 2
    assert _route(bad) == 1
    # hierarchical gating: groups divide E, k_primary divides k, per-level limits
    assert _route(_cfg(gating="hierarchical", E=16, k=4, groups=3, k_primary=2)) == 1
    assert _route(_cfg(gating="hierarchical", E=16, k=4, groups=4, k_primary=3)) == 1
    assert _route(_cfg(gating="hierarchical", E=16, k=4, groups=8, k_primary=1)) == 1  # 4 > b=2
    assert _route(_cfg(gating="hierarchical", E=16, k=8, groups=2, k_primary=1)) == 2  # 8 per group
    assert _route(_cfg(gating="hierarchical", E=256, k=4, groups=16, k_primary=2)) == 2  # 272 rows
    assert moe.lib.moe_route(None, FAKE, FAKE, None, None, None, FAKE, FAKE, None, None, None,
                             FAKE, None) == 1


def test_other_steps_validation():
    c = ctypes.byref(_cfg())
    P = FAKE
    assert moe.lib.moe_permute(c, None, P, P, P, P, P, P, P, None) == 1
    assert moe.lib.moe_permute(c, P, FAKE_ODD, P, P, P, P, P, P, None) == 1
    assert moe.lib.moe_expert_ffn(c, P, P, P, None, P, P, P, None) == 1
    assert moe.lib.moe_expert_ffn(c, P, P, P, P, FAKE_ODD, P, P, None) == 1
    assert moe.lib.moe_combine(c, P, None, P, P, P, None) == 1
    assert moe.lib.moe_combine(c, P, P, P, FAKE_ODD, P, None) == 1
    # the fused FFN + combine step: bf16 with k = 1, or k = 2 with an fp32 y; then the
    # usual argument checks
    c1 = ctypes.byref(_cfg(k=1))
    for bad in (_cfg(k=3), _cfg(k=2, y_bf16=True), _cfg(k=1, dtype="f32"), _cfg(k=2, dtype="f32")):
        assert moe.lib.moe_expert_ffn_combine(ctypes.byref(bad), P, P, P, P, P, P, P, P, P, P,
                                              None) == 2
        assert moe.lib.moe_expert_ffn_combine_gather(ctypes.byref(bad), P, P, P, P, P, P, P, P, P,
                                                     P, None) == 2
    assert moe.fused_combine(_cfg(k=1)) and moe.fused_combine(_cfg(k=2))
    assert not moe.fused_combine(_cfg(k=2, y_bf16=True)) and not moe.fused_combine(_cfg(k=4))
    assert moe.lib.moe_expert_ffn_combine(c1, P, P, None, P, P, P, P, P, P, P, None) == 1
    assert moe.lib.moe_expert_ffn_combine(c1, P, P, P, P, P, P, P, P, FAKE_ODD, P, None) == 1
    assert moe.lib.moe_forward(c, P, P, None, None, None, P, P, None, P, P, P, None, None, None,
                               P, None) == 1
    assert moe.lib.moe_get_error(None, None, None) == 1
    assert moe.lib.moe_wait_timeout_check(None, None) == 1
    assert moe.lib.moe_wait_timeout_check(FAKE_ODD, None) == 1


def test_workspace_sizes():
    c = _cfg()
    assert moe.moe_workspace_size(c) > 0
    assert moe.moe_forward_workspace_size(c) > moe.moe_workspace_size(c)
    assert moe.moe_workspace_size(_cfg(d_model=96)) == 0
    # the forward workspace holds x_perm, h (bf16) and y_perm (fp32) of T*k rows
    big = _cfg(T=16384, d_model=768, d_ff=3072, E=128, k=1)
    assert moe.moe_forward_workspace_size(big) >= 16384 * (768 * 2 + 3072 * 2 + 768 * 4)


def test_python_binding_rejects_cpu_tensors():
    import torch
    c = _cfg()
    x = torch.zeros(256, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        moe.moe_route(c, x, x, x, x, x)
