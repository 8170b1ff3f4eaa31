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


def pin_routed_scale_is_linear(mut):
    """The routed scale multiplies the normalised weights («Biased Routing»
    §"The router has two different scores": the factor is 1 for the
    checkpoint), so out - x scales with it exactly; a scale applied before
    the normalisation would cancel instead."""
    E, d, I, k = 6, 16, 8, 3
    layer = rand_layer(E, d, I, seed=81)
    x = rand_x(9, d, 81)
    o1 = oracle.forward(x, layer, k=k, eps=EPS, routed_scale=1.0, mutation=mut)["out"]
    o3 = oracle.forward(x, layer, k=k, eps=EPS, routed_scale=3.0, mutation=mut)["out"]
    xd = x.double().numpy()
    np.testing.assert_allclose(o3 - xd, 3.0 * (o1 - xd), rtol=1e-13, atol=1e-15)


def pin_margin(mut):
    """The margin c_(k) - c_(k+1) between the last selected and the best
    unselected biased score, which decides where the GPU selection must be
    exact. (a) A zero router gives s = 1/2 for every expert, so c = 1/2 + b and
    the margin is the gap between the k-th and (k+1)-th largest stored biases,
    exactly; (b) two biases tied at ranks k and k+1 give a margin of exactly
    0; (c) hand-set logits whose biased order differs from the unbiased one
    give the gap of the sorted biased scores; (d) random tokens: the gap
    between ranks k and k+1 of numpy's sort of s + b; (e) k = E gives inf."""
    d, E = 8, 8
    b = np.array([0.30, -0.10, 0.25, 0.05, -0.40, 0.125, 0.0, -0.2], np.float32)
    layer = {"norm_gain": torch.ones(d), "router_w": torch.zeros(E, d),
             "bias": torch.from_numpy(b)}
    x = torch.ones(1, d)
    r = oracle.route(x, layer, k=3, eps=EPS, mutation=mut)
    assert r["idx"][0].tolist() == [0, 2, 5], r["idx"][0]
    bd = b.astype(np.float64)
    want = (0.5 + bd[5]) - (0.5 + bd[3])          # exact in double
    assert r["margin"][0] == want, (r["margin"][0], want)
    b2 = b.copy()
    b2[3] = b2[5]                                   # tie at ranks 3 and 4
    r = oracle.route(x, dict(layer, bias=torch.from_numpy(b2)), k=3, eps=EPS, mutation=mut)
    assert r["idx"][0].tolist() == [0, 2, 3] and r["margin"][0] == 0.0, (r["idx"], r["margin"])
    # (c) logits 1.5, -2.25, 0, 3.75, -0.5, 0.125 with biases that reorder them
    E6 = 6
    l = torch.tensor([1.5, -2.25, 0.0, 3.75, -0.5, 0.125], dtype=torch.float64)
    b6 = torch.tensor([0.0, 0.6, 0.0, -0.5, 0.0, 0.3], dtype=torch.float32)
    layer6 = {"norm_gain": torch.ones(d), "router_w": (l / d)[:, None].expand(E6, d).float(),
              "bias": b6}
    r = oracle.route(x, layer6, k=2, eps=EPS, mutation=mut)
    c = torch.sigmoid(l / math.sqrt(1 + EPS)).numpy() + b6.double().numpy()
    # c ~ [0.818, 0.695, 0.5, 0.477, 0.378, 0.831]: experts 5, 0 selected, 1 next
    assert r["idx"][0].tolist() == [5, 0], r["idx"][0]
    np.testing.assert_allclose(r["margin"][0], c[0] - c[1], rtol=1e-12, atol=0)
    # (d) random tokens against a sort
    E, k = 16, 4
    layer = rand_layer(E, 32, 4, seed=23, bias_scale=0.2)
    rr = oracle.route(rand_x(60, 32, 23), layer, k=k, eps=EPS, mutation=mut)
    cs = -np.sort(-(rr["s"] + layer["bias"].double().numpy()[None, :]), axis=1)
    np.testing.assert_allclose(rr["margin"], cs[:, k - 1] - cs[:, k], rtol=1e-12, atol=1e-15)
    # (e) every expert selected: nothing to displace
    r = oracle.route(x, dict(layer6), k=E6, eps=EPS, mutation=mut)
    assert np.isinf(r["margin"][0])


def pin_forced_selection(mut):
    """A forced selection replaces the oracle's choice slot by slot, weights
    included: (a) forcing the oracle's own selection reproduces its output bit
    for bit; (b) forcing, per token, the three experts with the LOWEST biased
    scores in ascending order (never the oracle's choice, and not in its slot
    order) gives idx = the forced slots, w_j = s_f(j) / (sum_j s_f(j) + eps)
    and out = x + sum_j w_j SwiGLU_f(j)(xn), all written with
    torch.nn.functional in float64; (c) the forced rows follow the listed
    tokens, not the token ids."""
    E, d, I, k = 6, 16, 8, 3
    layer = rand_layer(E, d, I, seed=29, bias_scale=0.3)
    x = rand_x(5, d, 29)
    own = oracle.forward(x, layer, k=k, eps=EPS, mutation=mut)
    again = oracle.forward(x, layer, k=k, eps=EPS, forced=own["idx"], mutation=mut)
    assert np.array_equal(again["out"], own["out"]) and np.array_equal(again["idx"], own["idx"])
    # (b) an independent float64 computation of the forced mixture
    xd = x.double()
    xn = F.rms_norm(xd, (d,), weight=layer["norm_gain"].double(), eps=EPS)
    s = torch.sigmoid(xn @ layer["router_w"].double().T)
    c = s + layer["bias"].double()[None, :]
    forced = torch.argsort(c, dim=1)[:, :k].to(torch.int32)   # lowest c, ascending
    got = oracle.forward(x, layer, k=k, eps=EPS, forced=forced.numpy(), mutation=mut)
    assert np.array_equal(got["idx"], forced.numpy()), (got["idx"], forced)
    sf = torch.gather(s, 1, forced.long())
    w = sf / (sf.sum(1, keepdim=True) + EPS)
    np.testing.assert_allclose(got["w"], w.numpy(), rtol=1e-13, atol=0)
    want = xd.clone()
    for t in range(x.shape[0]):
        for j in range(k):
            e = int(forced[t, j])
            Wg, Wu = layer["w_gate_up"][e, :I].double(), layer["w_gate_up"][e, I:].double()
            y = F.linear(F.silu(F.linear(xn[t], Wg)) * F.linear(xn[t], Wu),
                         layer["w_down"][e].double())
            want[t] += w[t, j] * y
    np.testing.assert_allclose(got["out"], want.numpy(), rtol=1e-12, atol=1e-12)
    # (c) a token subset in another order, each with its own forced row
    toks = np.array([4, 1])
    sub = oracle.forward(x, layer, k=k, eps=EPS, tokens=toks, forced=forced.numpy()[toks],
                         mutation=mut)
    np.testing.assert_array_equal(sub["out"], got["out"][toks])


# ---------------------------------------------------------------- FP8_BLOCK
# "LFM2.5-24B-A2B: ein 24B-Reasoning-Modell, das pro Wortstück so wenig verbraucht wie ein 2B-Modell" (inferencekey.com,
# section "Für Engineers", paragraph "Quantisierung"): weights FP8 static in
# 128x128 blocks, activations FP8 dynamic per group of 128.

E4M3 = torch.float8_e4m3fn


def fp8_layer(E, d, I, seed, bias_scale=0.5):
    """A layer with e4m3 expert weights and per-block fp32 scales: codes of
    normal draws spread over the e4m3 range, scales around 1/(16 sqrt(K))."""
    base = rand_layer(E, d, I, seed, bias_scale=bias_scale)
    g = torch.Generator().manual_seed(seed + 7)
    return dict(
        base,
        w_gate_up=(torch.randn(E, 2 * I, d, generator=g) * 16).clamp(-448, 448).to(E4M3),
        w_down=(torch.randn(E, d, I, generator=g) * 16).clamp(-448, 448).to(E4M3),
        w_gate_up_scale=((0.5 + torch.rand(E, -(-2 * I // 128), -(-d // 128), generator=g))
                         / (16 * math.sqrt(d))).float(),
        w_down_scale=((0.5 + torch.rand(E, -(-d // 128), -(-I // 128), generator=g))
                      / (16 * math.sqrt(I))).float())


def dequant_weights(layer):
    """float64 weights = code value x block scale (torch's e4m3 decoding)."""
    def deq(codes, sc):
        full = sc.double().repeat_interleave(128, 1).repeat_interleave(128, 2)
        return codes.double() * full[:, :codes.shape[1], :codes.shape[2]]
    return dict(layer, w_gate_up=deq(layer["w_gate_up"], layer["w_gate_up_scale"]),
                w_down=deq(layer["w_down"], layer["w_down_scale"]))


def pin_e4m3_codec(mut):
    """The oracle's e4m3 decoding of all 256 codes and its encoding (nearest,
    ties to even, saturating) agree with torch's float8_e4m3fn conversions,
    on random values and on every midpoint between neighbouring codes."""
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes).view(E4M3).double().numpy()
    got = oracle.e4m3_value(codes)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan) and np.array_equal(got[~nan], want[~nan])
    pos = np.sort(want[:127])                      # 0 .. 448
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)  # exact in float
    g = torch.Generator().manual_seed(5)
    vals = np.concatenate([mids, -mids, pos.astype(np.float32),
                           (torch.randn(20000, generator=g) * 50).clamp(-460, 460).numpy(),
                           (torch.randn(5000, generator=g) * 0.01).numpy()]).astype(np.float32)
    ref = torch.from_numpy(vals).to(E4M3).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(vals)
    # torch writes -0 for negative values that round to zero; both are zero
    same = (got == ref) | ((got & 0x7F) == 0) & ((ref & 0x7F) == 0)
    assert same.all(), vals[~same][:5]


def pin_fp8_quant(mut):
    """Group quantisation: closed forms (a group at its amax maps to 448, a
    power-of-two amax gives exact codes, all-zero groups give zeros), groups
    of 128 quantised independently, and the rounding bound of e4m3 on random
    rows (relative 2^-4 for normal codes, 2^-10 s below)."""
    c = 0.125
    row = np.zeros(256)
    row[:6] = [448 * c, c, 0.5 * c, 1.0625 * c, -3 * c, 0.0]   # group 0: amax 448c
    row[128:130] = [0.3, 0.3]                                  # group 1: amax 0.3
    q = oracle.quant(row[None], mutation=mut)
    assert q["scales"][0, 0] == np.float32(c)
    np.testing.assert_array_equal(q["deq"][0, :6], [448 * c, c, 0.5 * c, c, -3 * c, 0.0])
    assert q["codes"][0, 0] == 0x7E and q["codes"][0, 128] == 0x7E
    assert q["scales"][0, 1] == np.float32(np.float32(0.3) / np.float32(448))
    z = oracle.quant(np.zeros((1, 130)), mutation=mut)
    assert not z["codes"].any() and not z["scales"].any() and not z["deq"].any()
    g = torch.Generator().manual_seed(6)
    v = (torch.randn(16, 384, generator=g) * torch.rand(16, 1, generator=g) * 3).double().numpy()
    q = oracle.quant(v, mutation=mut)
    s = np.repeat(q["scales"].astype(np.float64), 128, axis=1)
    amax = np.abs(v).reshape(16, 3, 128).max(2).repeat(128, 1)
    np.testing.assert_allclose(s, amax / 448, rtol=2e-7)
    err = np.abs(q["deq"] - v)
    assert (err <= np.maximum(np.abs(v) / 16, s * 2.0 ** -10) * (1 + 1e-6) + 1e-300).all()


def pin_fp8_expert_blocks(mut):
    """One expert with permutation weights, in closed form: gate row f holds
    code 1.0 and up row f code 2.0 at column (f + 128) mod 256, down is the
    identity; the 128x128 block scales all differ. Then G[f] = sg * xq[p(f)],
    U[f] = 2 su * xq[p(f)], y[j] = sd * Q(silu(G) U)[j], where xq = Q(x) and
    Q is the group quantisation (pinned by pin_fp8_quant), and sg, su, sd are
    the scales of the blocks the nonzero codes sit in."""
    d = I = 256
    perm = (np.arange(I) + 128) % d
    wgu = np.zeros((1, 2 * I, d), np.float32)
    wgu[0, np.arange(I), perm] = 1.0
    wgu[0, I + np.arange(I), perm] = 2.0
    wd = np.eye(d, dtype=np.float32)[None]
    sgu = np.array([[[0.5, 0.25], [2.0, 4.0], [1.0, 0.125], [8.0, 0.5]]], np.float32)
    sdn = np.array([[[2.0, 8.0], [0.25, 4.0]]], np.float32)
    layer = {"w_gate_up": torch.from_numpy(wgu).to(E4M3), "w_down": torch.from_numpy(wd).to(E4M3),
             "w_gate_up_scale": torch.from_numpy(sgu), "w_down_scale": torch.from_numpy(sdn)}
    g = torch.Generator().manual_seed(8)
    x = (torch.randn(3, d, generator=g) * 0.7).double().numpy()
    y = oracle.expert(x, layer, 0, mutation=mut)
    xq = oracle.quant(x)["deq"]
    rb = np.arange(I) // 128
    G = sgu[0, rb, 1 - rb] * xq[:, perm]
    U = 2 * sgu[0, 2 + rb, 1 - rb] * xq[:, perm]
    a = G * (1.0 / (1.0 + np.exp(-G))) * U
    want = sdn[0, rb, rb] * oracle.quant(a)["deq"]
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-300)


def pin_fp8_forward_error_bound(mut):
    """The FP8_BLOCK forward against the unquantised forward (pinned above) on
    the same, dequantised weights: the difference comes only from quantising
    the two expert inputs and stays inside its interval bound: per element
    |xq - xn| <= max(|xn|/16, s 2^-10) (plus the float rounding of xn),
    propagated through |Wg|, |Wu|, the SiLU's slope (below 1.1), the second
    quantisation and |Wd|, and weighted by the mixture weights."""
    E, d, I, k = 6, 256, 128, 2
    layer = fp8_layer(E, d, I, seed=51)
    ref = dequant_weights(layer)
    x = rand_x(12, d, 51)
    got = oracle.forward(x, layer, k=k, eps=EPS, mutation=mut)
    base = oracle.forward(x, ref, k=k, eps=EPS, forced=got["idx"])
    xn = oracle.rmsnorm(x, layer["norm_gain"], EPS)
    ex = np.maximum(np.abs(xn) / 16, np.abs(xn).reshape(12, 2, 128).max(2).repeat(128, 1)
                    / 448 * 2.0 ** -10) + np.abs(xn) * 2.0 ** -23
    bound = np.zeros((12, d))
    for t in range(12):
        for j, e in enumerate(got["idx"][t]):
            Wg, Wu = ref["w_gate_up"][e, :I].numpy(), ref["w_gate_up"][e, I:].numpy()
            Wd = ref["w_down"][e].numpy()
            G0, U0 = Wg @ xn[t], Wu @ xn[t]
            eG, eU = np.abs(Wg) @ ex[t], np.abs(Wu) @ ex[t]
            a0 = G0 / (1 + np.exp(-G0)) * U0
            da = 1.1 * eG * (np.abs(U0) + eU) + np.abs(G0 / (1 + np.exp(-G0))) * eU
            amax = np.abs(a0) + da
            sa = amax.reshape(1, 128).max(1).repeat(128) / 448
            ea = np.maximum(amax / 16, sa * 2.0 ** -10) + amax * 2.0 ** -23
            bound[t] += got["w"][t, j] * (np.abs(Wd) @ (da + ea))
    diff = np.abs(got["out"] - base["out"])
    assert (diff <= bound * 1.001 + 1e-12).all(), (diff / np.maximum(bound, 1e-30)).max()
    assert diff.max() > 0  # the quantisation does change the result


def pin_fp8_scale_code_trade(mut):
    """A block's scale and its codes trade a power of two exactly: doubling
    the scale of gate/up block (1, 0) of expert 2 while halving the codes
    inside that block (every code chosen with an exactly halvable value)
    leaves the output unchanged to the last bit."""
    E, d, I, k = 3, 256, 128, 3
    layer = fp8_layer(E, d, I, seed=61)
    v = layer["w_gate_up"].float()
    v = torch.where(v.abs() < 2.0 ** -5, torch.full_like(v, 0.25), v)  # normal, halvable
    layer["w_gate_up"] = v.to(E4M3)
    x = rand_x(4, d, 61)
    o0 = oracle.forward(x, layer, k=k, eps=EPS, mutation=mut)["out"]
    l2 = dict(layer)
    wgu = layer["w_gate_up"].float().clone()
    wgu[2, 128:256, 0:128] /= 2
    l2["w_gate_up"] = wgu.to(E4M3)
    sc = layer["w_gate_up_scale"].clone()
    sc[2, 1, 0] *= 2
    l2["w_gate_up_scale"] = sc
    assert torch.equal(l2["w_gate_up"].float()[2, 128:256, :128] * 2,
                       layer["w_gate_up"].float()[2, 128:256, :128])
    o1 = oracle.forward(x, l2, k=k, eps=EPS, mutation=mut)["out"]
    np.testing.assert_array_equal(o0, o1)


def pin_fp8_sign_symmetry(mut):
    """Quantisation is odd: negating a row flips every code's sign bit (zero
    codes excepted) and keeps the scales; the dequantised row is negated."""
    g = torch.Generator().manual_seed(9)
    v = (torch.randn(4, 256, generator=g) * 2).double().numpy()
    a, b = oracle.quant(v, mutation=mut), oracle.quant(-v, mutation=mut)
    np.testing.assert_array_equal(a["scales"], b["scales"])
    nz = (a["codes"] & 0x7F) != 0
    np.testing.assert_array_equal(a["codes"][nz] ^ 0x80, b["codes"][nz])
    np.testing.assert_array_equal(a["deq"], -b["deq"])


def pin_fp8_zero_block_scale(mut):
    """A block scale of zero removes exactly that block: the output equals the
    one with the block's codes set to zero (both leave the other 127 x 128
    blocks' products untouched, and a scale read from the wrong block would
    change a different block)."""
    E, d, I, k = 2, 256, 128, 2
    layer = fp8_layer(E, d, I, seed=71)
    x = rand_x(5, d, 71)
    a = dict(layer)
    sc = layer["w_gate_up_scale"].clone()
    sc[1, 0, 1] = 0.0
    a["w_gate_up_scale"] = sc
    b = dict(layer)
    wgu = layer["w_gate_up"].float().clone()
    wgu[1, 0:128, 128:256] = 0.0
    b["w_gate_up"] = wgu.to(E4M3)
    oa = oracle.forward(x, a, k=k, eps=EPS, mutation=mut)["out"]
    ob = oracle.forward(x, b, k=k, eps=EPS, mutation=mut)["out"]
    np.testing.assert_array_equal(oa, ob)
    o0 = oracle.forward(x, layer, k=k, eps=EPS, mutation=mut)["out"]
    assert np.abs(oa - o0).max() > 0


# ------------------------------------------------- neighbouring steps of the block
# «Biased Routing» §"The exact checkpoint" (the first two layers are dense and
# convolutional; pre-norm and a residual around mixer and feed-forward) and
# §"A short convolution is a local mixer, not an embedding lookup".

def conv_layer(d, seed, dtype=torch.float32):
    g = torch.Generator().manual_seed(seed)
    return {"norm_gain": (1 + 0.1 * torch.randn(d, generator=g)).float(),
            "w_in": (torch.randn(3 * d, d, generator=g) / math.sqrt(d)).to(dtype),
            "w_out": (torch.randn(d, d, generator=g) / math.sqrt(d)).to(dtype),
            "conv": torch.randn(d, 3, generator=g).float()}


def conv_textbook(x, layer, eps=EPS, state=None):
    """The block with torch.nn.functional in float64: rms_norm, one linear for
    the three streams, a depthwise conv1d (weights reversed: conv1d's tap j
    multiplies position t - 2 + j, i.e. lag 2 - j), a linear back."""
    B, T, d = x.shape
    xn = F.rms_norm(x.double(), (d,), weight=layer["norm_gain"].double(), eps=eps)
    g, u, v = F.linear(xn, layer["w_in"].double()).split(d, dim=-1)
    a = (g * v).transpose(1, 2)                              # [B, d, T]
    hist = torch.zeros(B, d, 2, dtype=torch.float64) if state is None else \
        torch.as_tensor(state).double().transpose(1, 2)
    a = torch.cat([hist, a], dim=2)                          # positions -2 .. T-1
    c = F.conv1d(a, layer["conv"].double().flip(1)[:, None, :], groups=d)   # [B, d, T]
    y = u * c.transpose(1, 2)
    return (x.double() + F.linear(y, layer["w_out"].double())).numpy()


def pin_dense_ffn(mut):
    """Dense feed-forward block = x + SwiGLU(RMSNorm(x)) written with
    torch.nn.functional in float64; W_down = 0 gives x exactly."""
    d, I = 24, 40
    g = torch.Generator().manual_seed(13)
    layer = {"norm_gain": (1 + 0.1 * torch.randn(d, generator=g)).float(),
             "w_gate_up": (torch.randn(2 * I, d, generator=g) / math.sqrt(d)).float(),
             "w_down": (torch.randn(d, I, generator=g) / math.sqrt(I)).float()}
    x = rand_x(9, d, 13)
    out = oracle.dense_ffn(x, layer, EPS, mutation=mut)
    xn = F.rms_norm(x.double(), (d,), weight=layer["norm_gain"].double(), eps=EPS)
    Wg, Wu = layer["w_gate_up"][:I].double(), layer["w_gate_up"][I:].double()
    want = x.double() + F.linear(F.silu(F.linear(xn, Wg)) * F.linear(xn, Wu),
                                 layer["w_down"].double())
    np.testing.assert_allclose(out, want.numpy(), rtol=1e-12, atol=1e-12)
    z = dict(layer, w_down=torch.zeros_like(layer["w_down"]))
    assert np.array_equal(oracle.dense_ffn(x, z, EPS, mutation=mut), x.double().numpy())


def pin_shortconv_textbook(mut):
    """The short-convolution block against its torch.nn.functional form, with
    and without a carried state, on two sequences."""
    d, B, T = 12, 2, 7
    layer = conv_layer(d, 17)
    x = torch.randn(B, T, d, generator=torch.Generator().manual_seed(18))
    out, _ = oracle.shortconv(x, layer, EPS, mutation=mut)
    np.testing.assert_allclose(out, conv_textbook(x, layer), rtol=1e-11, atol=1e-12)
    st = np.random.default_rng(19).normal(size=(B, 2, d))
    out, _ = oracle.shortconv(x, layer, EPS, state_in=st, mutation=mut)
    np.testing.assert_allclose(out, conv_textbook(x, layer, state=st), rtol=1e-11, atol=1e-12)


def pin_shortconv_delta_kernels(mut):
    """Closed forms: a delta kernel at lag 0 makes the block position-wise,
    x + W_out (u g v); a delta at lag 1 is the identity shift, c_t = a_{t-1}
    (zero before the sequence); zero u rows give out = x exactly."""
    d, B, T = 8, 1, 6
    layer = conv_layer(d, 21)
    x = torch.randn(B, T, d, generator=torch.Generator().manual_seed(22))
    xn = F.rms_norm(x.double(), (d,), weight=layer["norm_gain"].double(), eps=EPS)
    g, u, v = F.linear(xn, layer["w_in"].double()).split(d, dim=-1)
    Wo = layer["w_out"].double()
    for lag in (0, 1):
        k = torch.zeros(d, 3)
        k[:, lag] = 1.0
        out, _ = oracle.shortconv(x, dict(layer, conv=k), EPS, mutation=mut)
        a = g * v
        if lag == 1:
            a = torch.cat([torch.zeros(B, 1, d, dtype=torch.float64), a[:, :-1]], dim=1)
        want = x.double() + F.linear(u * a, Wo)
        np.testing.assert_allclose(out, want.numpy(), rtol=1e-12, atol=1e-12)
    w_in = layer["w_in"].clone()
    w_in[d:2 * d] = 0.0
    out, _ = oracle.shortconv(x, dict(layer, w_in=w_in), EPS, mutation=mut)
    assert np.array_equal(out, x.double().numpy())


def pin_shortconv_causal(mut):
    """Receptive field of three positions, causal, per sequence: changing one
    token changes only its own output and the next two, and no other
    sequence of the batch."""
    d, B, T = 8, 2, 9
    layer = conv_layer(d, 23)
    x = torch.randn(B, T, d, generator=torch.Generator().manual_seed(24))
    o0, _ = oracle.shortconv(x, layer, EPS, mutation=mut)
    for tp in (3, T - 1):
        x2 = x.clone()
        x2[0, tp] += 1.0
        o1, _ = oracle.shortconv(x2, layer, EPS, mutation=mut)
        changed = np.abs(o1 - o0).max(axis=2) > 0
        want = np.zeros((B, T), bool)
        want[0, tp:min(T, tp + 3)] = True
        assert np.array_equal(changed, want), (tp, changed)


def pin_shortconv_state_chaining(mut):
    """Running T1 then T2 positions with the state carried equals running
    T1 + T2 at once, outputs and final state bit for bit; decode (T = 1
    steps) too."""
    d, B, T = 8, 2, 7
    layer = conv_layer(d, 25)
    x = torch.randn(B, T, d, generator=torch.Generator().manual_seed(26))
    full, s_full = oracle.shortconv(x, layer, EPS, mutation=mut)
    a, s = oracle.shortconv(x[:, :4].contiguous(), layer, EPS, mutation=mut)
    b, s2 = oracle.shortconv(x[:, 4:].contiguous(), layer, EPS, state_in=s, mutation=mut)
    assert np.array_equal(np.concatenate([a, b], 1), full) and np.array_equal(s2, s_full)
    st, outs = None, []
    for t in range(T):
        o, st = oracle.shortconv(x[:, t:t + 1].contiguous(), layer, EPS, state_in=st, mutation=mut)
        outs.append(o)
    assert np.array_equal(np.concatenate(outs, 1), full) and np.array_equal(st, s_full)


PINS = [pin_five_candidate, pin_rmsnorm, pin_router_sigmoid, pin_weights_sum_below_one,
        pin_k1, pin_tie_break, pin_brute_force_subsets, pin_zero_bias_is_logit_topk,
        pin_bias_shift_invariance, pin_all_selected_bias_invariance,
        pin_zero_down_is_identity, pin_identical_experts, pin_routed_scale_is_linear,
        pin_margin, pin_forced_selection, pin_e4m3_codec, pin_fp8_quant,
        pin_fp8_expert_blocks, pin_fp8_forward_error_bound, pin_fp8_scale_code_trade,
        pin_fp8_sign_symmetry, pin_fp8_zero_block_scale,
        pin_dense_ffn, pin_shortconv_textbook, pin_shortconv_delta_kernels,
        pin_shortconv_causal, pin_shortconv_state_chaining]
