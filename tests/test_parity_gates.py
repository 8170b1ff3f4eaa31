"""The GPU parity gates themselves, on the CPU: outputs that differ from the
oracle only by the storage rounding pass; a MoE part off by a few percent,
which the bound on out alone would let through because the residual
dominates ||out||, fails."""
import numpy as np
import pytest
import torch

import oracle
from sigmoid_bias_top_b200 import workloads as W
from tests import parity as PA


@pytest.fixture(scope="module")
def decode8():
    w = W.DECODE.scaled(n_tokens=8)
    layer = PA.to_cpu_layer(W.make_layer(w, 0, "cpu"))
    x = W.make_x(w, "cpu")
    r = oracle.route(x, layer, w.top_k, w.eps, w.routed_scale)
    ref = oracle.forward(x, layer, w.top_k, w.eps, w.routed_scale, forced=r["idx"])
    return w, layer, x, r["idx"], ref["out"]


def test_storage_rounding_passes(decode8):
    w, layer, x, idx, ref = decode8
    out = torch.from_numpy(ref).to(torch.bfloat16)
    err, derr = PA.check_outputs(x, layer, w.top_k, w.eps, w.routed_scale, out, idx,
                                 np.arange(8), "bf16")
    assert err < 4e-3 and derr < 2e-2


@pytest.mark.parametrize("factor", [1.03, 0.96])
def test_scaled_moe_part_fails(decode8, factor):
    """out = x + factor * MoE(x), rounded to bf16: within 1e-2 of ||out|| on
    every token (the residual dominates), but 3-4% off in the MoE part."""
    w, layer, x, idx, ref = decode8
    xd = x.double().numpy()
    fake = xd + factor * (ref - xd)
    rel = np.linalg.norm(fake - ref, axis=1) / np.linalg.norm(ref, axis=1)
    assert rel.max() < PA.TOL["bf16"]          # the out gate alone would pass it
    with pytest.raises(AssertionError, match="MoE-delta"):
        PA.check_outputs(x, layer, w.top_k, w.eps, w.routed_scale,
                         torch.from_numpy(fake).to(torch.bfloat16), idx, np.arange(8), "bf16")


def test_dropped_slot_fails(decode8):
    """The last slot's expert output left out of the sum."""
    w, layer, x, idx, ref = decode8
    part = oracle.forward(x, layer, w.top_k, w.eps, w.routed_scale, forced=idx)
    xn = oracle.rmsnorm(x, layer["norm_gain"], w.eps)
    fake = ref.copy()
    for t in range(8):
        e = int(idx[t, -1])
        fake[t] -= part["w"][t, -1] * oracle.expert(xn[t:t + 1], layer, e)[0]
    with pytest.raises(AssertionError):
        PA.check_outputs(x, layer, w.top_k, w.eps, w.routed_scale,
                         torch.from_numpy(fake).to(torch.bfloat16), idx, np.arange(8), "bf16")


def test_near_tie_bound_counts_margins():
    """A batch where every token is a near tie (all biases equal and a zero
    router: every margin is 0) is refused by the near-tie bound."""
    E, d, k, N = 8, 16, 2, 20
    layer = {"norm_gain": torch.ones(d), "router_w": torch.zeros(E, d), "bias": torch.zeros(E)}
    x = torch.randn(N, d, generator=torch.Generator().manual_seed(3))
    r_gpu = {"idx": torch.tensor([[0, 1]] * N, dtype=torch.int32),
             "w": torch.full((N, k), 0.5 / (1.0 + 1e-6))}
    with pytest.raises(AssertionError, match="near ties"):
        PA.check_routing(x, layer, k, 1e-6, 1.0, r_gpu)
