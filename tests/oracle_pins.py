"""Pins of the fp64 oracle against what the page and the mathematics fix.

Each pin takes `mut` (a planted-mistake code of the oracle, 0 = the method)
and raises AssertionError when the oracle disagrees with the fixed result.
tests/test_oracle_pins.py runs every pin on the unmodified oracle, and checks
that every planted mistake is caught by at least one pin.

Source page: "LFM2.5-24B-A2B: Biased Routing, Short Convolutions and Ten KV
Caches" (flozi.net, English page).
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
EPS = 1e-6


def rand_layer(E, d, I, seed, bias_scale=0.5, dtype=torch.float32, gain_jitter=0.1):
    g = torch.Generator().manual_seed(seed)
    return {
        "norm_gain": (1 + gain_jitter * torch.randn(d, generator=g)).float(),
        "router_w": (torch.randn(E, d, generator=g) / math.sqrt(d)).float(),
        "bias": ((torch.rand(E, generator=g) * 2 - 1) * bias_scale).float(),
        "w_gate_up": (torch.randn(E, 2 * I, d, generator=g) / math.sqrt(d)).to(dtype),
        "w_down": (torch.randn(E, d, I, generator=g) / math.sqrt(I)).to(dtype),
    }


def rand_x(N, d, seed, dtype=torch.float32):
    g = torch.Generator().manual_seed(seed + 100)
    return torch.randn(N, d, generator=g).to(dtype)


def five_candidate_case(d=16):
    """One token built so that its unbiased scores are the golden ones."""
    gold = json.load(open(os.path.join(GOLDEN, "five_candidate.json")))
    E = gold["fixed_by_page"]["n_experts"]
    s = np.zeros(E)
    lo, hi = gold["others_unbiased_range"]
    s[:] = np.linspace(lo, hi, E)
    b = np.zeros(E)
    for name, e in gold["experts"].items():
        s[e] = gold["unbiased"][name]
        b[e] = gold["bias"][name]
    logit = np.log(s / (1 - s))
    # x = 1, gain = 1: xn_j = 1/sqrt(1+eps), so l_e = d * W_r[e, j] / sqrt(1 + eps)
    rw = torch.tensor(np.repeat((logit * math.sqrt(1 + EPS) / d)[:, None], d, 1),
                      dtype=torch.float32)
    I = 8
    g = torch.Generator().manual_seed(5)
    layer = {"norm_gain": torch.ones(d), "router_w": rw,
             "bias": torch.tensor(b, dtype=torch.float32),
             "w_gate_up": torch.randn(E, 2 * I, d, generator=g) / 4,
             "w_down": torch.randn(E, d, I, generator=g) / 3}
    return gold, torch.ones(1, d), layer


def pin_five_candidate(mut):
    """E displaces D yet contributes with 0.40, not its biased 0.60."""
    gold, x, layer = five_candidate_case()
    r = oracle.route(x, layer, k=4, eps=EPS, mutation=mut)
    want = [gold["experts"][n] for n in gold["expected_slots"]]
    assert r["idx"][0].tolist() == want, (r["idx"][0], want)
    u = gold["unbiased"]
    S = sum(u[n] for n in gold["expected_slots"])
    w_want = np.array([u[n] / (S + EPS) for n in gold["expected_slots"]])
    np.testing.assert_allclose(r["w"][0], w_want, rtol=1e-6, atol=0)
    # the displaced expert's coefficient comes from 0.40, not the biased 0.60
    wE = r["w"][0][3]
    assert abs(wE - 0.40 / (S + EPS)) < 1e-6
    assert abs(wE - gold["fixed_by_page"]["E_biased"] / (S + 0.2 + EPS)) > 1e-2


def pin_rmsnorm(mut):
    """Constant rows a*1 give a/sqrt(a^2+eps)*g; zero rows give 0; random rows
    match torch's rms_norm in float64."""
    d = 24
    g = torch.Generator().manual_seed(11)
    gain = (1 + 0.3 * torch.randn(d, generator=g)).float()
    a = torch.tensor([0.5, -2.0, 3e-4, 7.0], dtype=torch.float64)
    x = torch.cat([a[:, None].expand(4, d), torch.zeros(1, d)]).float()
    xn = oracle.rmsnorm(x, gain, EPS, mutation=mut)
    a = x[:4, 0].double()                      # the values as stored
    want = (a / torch.sqrt(a * a + EPS))[:, None] * gain.double()[None, :]
    np.testing.assert_allclose(xn[:4], want.numpy(), rtol=1e-13, atol=0)
    assert np.all(xn[4] == 0.0)
    xr = rand_x(6, d, 3)
    ref = F.rms_norm(xr.double(), (d,), weight=gain.double(), eps=EPS)
    np.testing.assert_allclose(oracle.rmsnorm(xr, gain, EPS, mutation=mut), ref.numpy(),
                               rtol=1e-12, atol=1e-14)


def pin_router_sigmoid(mut):
    """x = 1 and hand-set router rows give chosen logits; s = sigmoid(l)."""
    d, E = 8, 6
    l = torch.tensor([1.5, -2.25, 0.0, 3.75, -0.5, 0.125], dtype=torch.float64)
    layer = {"norm_gain": torch.ones(d), "router_w": (l / d)[:, None].expand(E, d).float(),
             "bias": torch.zeros(E)}
    r = oracle.route(torch.ones(1, d), layer, k=2, eps=EPS, mutation=mut)
    want = torch.sigmoid(l / math.sqrt(1 + EPS))
    np.testing.assert_allclose(r["s"][0], want.numpy(), rtol=1e-14, atol=0)


def pin_weights_sum_below_one(mut):
    """sum_j w_j = S/(S+eps) < 1 in exact arithmetic."""
    layer = rand_layer(16, 32, 8, seed=21)
    r = oracle.route(rand_x(64, 32, 21), layer, k=4, eps=EPS, mutation=mut)
    S = np.take_along_axis(r["s"], r["idx"].astype(np.int64), 1).sum(1)
    gap = 1.0 - r["w"].sum(1)
    assert np.all(gap > 0), gap.min()
    np.testing.assert_allclose(gap, EPS / (S + EPS), rtol=1e-6, atol=0)


def pin_k1(mut):
    """k = 1: the single weight is s/(s+eps)."""
    layer = rand_layer(8, 16, 8, seed=31)
    r = oracle.route(rand_x(20, 16, 31), layer, k=1, eps=EPS, mutation=mut)
    s = np.take_along_axis(r["s"], r["idx"].astype(np.int64), 1)[:, 0]
    np.testing.assert_allclose(r["w"][:, 0], s / (s + EPS), rtol=1e-14, atol=0)


def pin_tie_break(mut):
    """Exactly tied biased scores: the lower expert index takes the earlier slot."""
    d, E = 8, 8
    l = torch.tensor([0.0, -1.0, 2.0, -0.5, 0.25, 2.0, -3.0, 1.0], dtype=torch.float64)
    layer = {"norm_gain": torch.ones(d), "router_w": (l / d)[:, None].expand(E, d).float(),
             "bias": torch.zeros(E)}
    x = torch.ones(1, d)
    assert oracle.route(x, layer, k=1, eps=EPS, mutation=mut)["idx"][0].tolist() == [2]
    assert oracle.route(x, layer, k=3, eps=EPS, mutation=mut)["idx"][0].tolist() == [2, 5, 7]


def pin_brute_force_subsets(mut):
    """For E = 12, k = 4 the selected set maximises the sum of s + b over all
    C(12, 4) subsets, and slots are in descending s + b."""
    E, k = 12, 4
    layer = rand_layer(E, 16, 4, seed=41, bias_scale=0.3)
    r = oracle.route(rand_x(40, 16, 41), layer, k=k, eps=EPS, mutation=mut)
    b = layer["bias"].double().numpy()
    for t in range(40):
        c = r["s"][t] + b
        best = max(itertools.combinations(range(E), k), key=lambda S: sum(c[list(S)]))
        assert set(best) == set(r["idx"][t].tolist()), t
        cs = c[r["idx"][t]]
        assert np.all(np.diff(cs) <= 0), cs


def pin_zero_bias_is_logit_topk(mut):
    """With zero bias the selection equals the top-k logits (sigmoid is monotone)."""
    E, d, k = 16, 32, 4
    layer = rand_layer(E, d, 4, seed=51)
    layer["bias"] = torch.zeros(E)
    x = rand_x(50, d, 51)
    r = oracle.route(x, layer, k=k, eps=EPS, mutation=mut)
    logits = oracle.rmsnorm(x, layer["norm_gain"], EPS) @ layer["router_w"].double().numpy().T
    want = np.argsort(-logits, axis=1, kind="stable")[:, :k]
    np.testing.assert_array_equal(r["idx"], want)


def pin_bias_shift_invariance(mut):
    """Adding one constant to every bias leaves the selection unchanged."""
    layer = rand_layer(16, 32, 4, seed=61)
    x = rand_x(50, 32, 61)
    r0 = oracle.route(x, layer, k=4, eps=EPS, mutation=mut)
    l2 = dict(layer, bias=layer["bias"] + 0.25)
    r1 = oracle.route(x, l2, k=4, eps=EPS, mutation=mut)
    np.testing.assert_array_equal(r0["idx"], r1["idx"])
    np.testing.assert_array_equal(r0["w"], r1["w"])


def pin_all_selected_bias_invariance(mut):
    """k = E: every expert is selected, so the output does not depend on the bias."""
    E = 6
    layer = rand_layer(E, 24, 16, seed=71, bias_scale=0.8)
    x = rand_x(12, 24, 71)
    o0 = oracle.forward(x, layer, k=E, eps=EPS, mutation=mut)["out"]
    l2 = dict(layer, bias=-layer["bias"] * 3)
    o1 = oracle.forward(x, l2, k=E, eps=EPS, mutation=mut)["out"]
    np.testing.assert_allclose(o0, o1, rtol=1e-12, atol=1e-12)


def pin_zero_down_is_identity(mut):
    """W_down = 0: the block returns its input exactly."""
    layer = rand_layer(8, 24, 16, seed=81)
    layer["w_down"] = torch.zeros_like(layer["w_down"])
    x = rand_x(10, 24, 81)
    out = oracle.forward(x, layer, k=2, eps=EPS, mutation=mut)["out"]
    assert np.array_equal(out, x.double().numpy())


def pin_identical_experts(mut):
    """All experts equal: out = x + S/(S+eps) * SwiGLU(xn), the SwiGLU written
    with torch.nn.functional in float64."""
    E, d, I, k = 5, 24, 16, 3
    base = rand_layer(1, d, I, seed=91)
    layer = dict(base, router_w=rand_layer(E, d, I, seed=92)["router_w"],
                 bias=rand_layer(E, d, I, seed=93)["bias"],
                 w_gate_up=base["w_gate_up"].expand(E, 2 * I, d).contiguous(),
                 w_down=base["w_down"].expand(E, d, I).contiguous())
    x = rand_x(7, d, 91)
    res = oracle.forward(x, layer, k=k, eps=EPS, mutation=mut)
    r = oracle.route(x, layer, k=k, eps=EPS)
    S = np.take_along_axis(r["s"], r["idx"].astype(np.int64), 1).sum(1)
    xn = torch.tensor(oracle.rmsnorm(x, layer["norm_gain"], EPS))
    Wg, Wu = base["w_gate_up"][0, :I].double(), base["w_gate_up"][0, I:].double()
    Wd = base["w_down"][0].double()
    mlp = F.linear(F.silu(F.linear(xn, Wg)) * F.linear(xn, Wu), Wd)
    want = x.double() + torch.tensor(S / (S + EPS))[:, None] * mlp
    np.testing.assert_allclose(res["out"], want.numpy(), rtol=1e-12, atol=1e-12)


PINS = [pin_five_candidate, pin_rmsnorm, pin_router_sigmoid, pin_weights_sum_below_one,
        pin_k1, pin_tie_break, pin_brute_force_subsets, pin_zero_bias_is_logit_topk,
        pin_bias_shift_invariance, pin_all_selected_bias_invariance,
        pin_zero_down_is_identity, pin_identical_experts]
