"""The synthetic workloads have the structure their descriptions ask for,
checked with the oracle's routing on CPU-drawn inputs."""
import numpy as np
import torch

import oracle
from sigmoid_bias_top_b200 import workloads as W


def _route(w, layer, x, **kw):
    return oracle.route(x, layer, w.top_k, w.eps, w.routed_scale, **kw)


def test_tiny_bias_changes_at_least_five_selections():
    w = W.TINY_F32
    x, layers = W.make_inputs(w)
    r = _route(w, layers[0], x)
    nob = dict(layers[0], bias=torch.zeros_like(layers[0]["bias"]))
    r0 = _route(w, nob, x)
    changed = sum(set(a) != set(b) for a, b in zip(r["idx"].tolist(), r0["idx"].tolist()))
    assert changed >= 5, changed


def test_decode_activates_most_experts():
    w = W.DECODE
    layer = W.make_layer(w, with_experts=False)
    r = _route(w, layer, W.make_x(w))
    active = np.unique(r["idx"]).size
    assert 45 <= active <= 64, active


def test_prefill_is_near_uniform():
    w = W.PREFILL.scaled(n_tokens=4096)
    layer = W.make_layer(w, with_experts=False)
    assert float(layer["bias"].abs().max()) == 0.0
    r = _route(w, layer, W.make_x(w))
    counts = np.bincount(r["idx"].reshape(-1), minlength=64)
    mean = counts.mean()
    assert counts.min() > 0.6 * mean and counts.max() < 1.5 * mean, counts


def test_skewed_load_profile():
    """Top 8 experts take about half of the 65,536 assignments; at least 4
    experts get fewer than 16 tokens."""
    w = W.SKEWED
    layer = W.make_layer(w, with_experts=False)
    r = _route(w, layer, W.make_x(w))
    counts = np.bincount(r["idx"].reshape(-1), minlength=64)
    assert counts.sum() == 65536
    top8 = np.sort(counts)[::-1][:8].sum() / counts.sum()
    assert 0.4 <= top8 <= 0.6, top8
    assert (counts < 16).sum() >= 4, np.sort(counts)[:8]


def test_generator_is_seeded():
    a = W.make_x(W.DECODE)
    b = W.make_x(W.DECODE)
    assert torch.equal(a, b)
    l0 = W.make_layer(W.TINY_F32, 0)
    l1 = W.make_layer(W.TINY_F32, 1)
    assert not torch.equal(l0["router_w"], l1["router_w"])
    assert torch.equal(W.make_layer(W.TINY_F32, 0, with_experts=False)["router_w"],
                       l0["router_w"])


def test_verify_widens_the_expert_union():
    """320 verify tokens (32 sequences x 10) activate (nearly) every expert,
    more than the 32-token decode step."""
    w = W.VERIFY
    layer = W.make_layer(w, with_experts=False)
    r = _route(w, layer, W.make_x(w))
    active = np.unique(r["idx"]).size
    wd = W.DECODE
    rd = _route(wd, W.make_layer(wd, with_experts=False), W.make_x(wd))
    assert active >= 62 and active > np.unique(rd["idx"]).size, active


def test_fp8_layer_draw():
    """FP8_BLOCK layers: e4m3 expert matrices, one fp32 scale per 128x128
    block, the dequantised weights at the bf16 workloads' standard deviation,
    the same router tensors as a draw without experts."""
    w = W.DECODE_FP8.scaled(n_experts=4, d=256, d_ff=384)
    layer = W.make_layer(w, 0)
    assert layer["w_gate_up"].dtype == torch.float8_e4m3fn
    assert layer["w_down"].dtype == torch.float8_e4m3fn
    assert tuple(layer["w_gate_up_scale"].shape) == (4, 6, 2)
    assert tuple(layer["w_down_scale"].shape) == (4, 2, 3)
    sc = layer["w_gate_up_scale"].repeat_interleave(128, 1).repeat_interleave(128, 2)
    deq = layer["w_gate_up"].float() * sc
    assert abs(deq.std().item() - w.gate_up_std) < 0.05 * w.gate_up_std
    assert not torch.isnan(layer["w_down"].float()).any()
    r = W.make_layer(w, 0, with_experts=False)
    assert torch.equal(r["router_w"], layer["router_w"]) and torch.equal(r["bias"], layer["bias"])
