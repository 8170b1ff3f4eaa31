"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on the five
workloads and on edge cases. Needs an sm_100 GPU."""
import numpy as np
import pytest
import torch

from sigmoid_bias_top_b200 import MoeError, MoeLayer, workloads as W
from tests import parity as PA

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run(w, x=None, layer=None, max_tokens=None, layer_idx=0):
    if layer is None:
        layer = W.make_layer(w, layer_idx, DEV)
    if x is None:
        x = W.make_x(w, DEV)
    N = x.shape[0]
    m = MoeLayer(layer, w.top_k, w.eps, w.routed_scale, max_tokens=max_tokens or max(N, 1))
    out = m(x)
    torch.cuda.synchronize()
    assert m.status() == 0
    r = m.debug_routing(N)
    torch.cuda.synchronize()
    return m, x, layer, out, r


def full_check(w, x, layer, out, r, tokens=None):
    x_cpu, l_cpu = x.cpu(), PA.to_cpu_layer(layer)
    ref, idx, n_near = PA.check_routing(x_cpu, l_cpu, w.top_k, w.eps, w.routed_scale, r)
    d = PA.check_dispatch(idx, w.n_experts, r)
    if tokens is None:
        tokens = np.arange(x.shape[0])
    elif isinstance(tokens, str):
        tokens = PA.sample_tokens(x.shape[0], idx, d["offsets"], n_random=128)
    err, derr = PA.check_outputs(x_cpu, l_cpu, w.top_k, w.eps, w.routed_scale, out, idx,
                                 tokens, w.dtype)
    return {"err": err, "delta_err": derr, "near_ties": n_near, "counts": d["counts"]}


def test_tiny_f32_full():
    w = W.TINY_F32
    m, x, layer, out, r = run(w)
    full_check(w, x, layer, out, r)


def test_decode_full():
    w = W.DECODE
    m, x, layer, out, r = run(w)
    res = full_check(w, x, layer, out, r)
    assert (res["counts"] > 0).sum() >= 45


def test_verify_sampled():
    """The 320-token speculative verify step (fused expert kernel, all experts)."""
    w = W.VERIFY
    m, x, layer, out, r = run(w)
    assert m.launches_per_forward(w.n_tokens) == 4
    res = full_check(w, x, layer, out, r, tokens="sample")
    assert (res["counts"] > 0).sum() >= 62


def test_prefill_sampled():
    w = W.PREFILL
    m, x, layer, out, r = run(w)
    full_check(w, x, layer, out, r, tokens="sample")


def test_skewed_sampled():
    w = W.SKEWED
    m, x, layer, out, r = run(w)
    res = full_check(w, x, layer, out, r, tokens="sample")
    c = np.sort(res["counts"])[::-1]
    assert 0.4 <= c[:8].sum() / c.sum() <= 0.6
    assert (res["counts"] < 16).sum() >= 4


def test_stacked_decode_every_block_routing():
    """38 chained blocks h = x + MoE(RMSNorm(x)); every block's routing checked
    against the oracle on that block's GPU input (teacher forcing), outputs of
    blocks 1, 19 and 38 checked on sampled tokens."""
    w = W.STACKED
    x = W.make_x(w, DEV)
    out_blocks = {0, 18, 37}
    for l in range(w.n_layers):
        layer = W.make_layer(w, l, DEV)
        m = MoeLayer(layer, w.top_k, w.eps, w.routed_scale, max_tokens=w.n_tokens)
        y = m(x)
        torch.cuda.synchronize()
        assert m.status() == 0
        r = m.debug_routing(w.n_tokens)
        x_cpu = x.cpu()
        l_cpu = {k: v.cpu() for k, v in layer.items() if k in ("norm_gain", "router_w", "bias")}
        ref, idx, _ = PA.check_routing(x_cpu, l_cpu, w.top_k, w.eps, w.routed_scale, r)
        PA.check_dispatch(idx, w.n_experts, r)
        if l in out_blocks:
            toks = np.random.default_rng(l).choice(w.n_tokens, 24, replace=False)
            PA.check_outputs(x_cpu, PA.to_cpu_layer(layer), w.top_k, w.eps, w.routed_scale,
                             y, idx, toks, w.dtype)
        m.close()
        del layer
        x = y


SMALL_BF16 = W.Workload(name="small_bf16", n_tokens=300, d=320, n_experts=16, top_k=4,
                        d_ff=320, dtype="bf16", seed=11, gain_jitter=0.02, router_std=0.06,
                        bias_kind="uniform", bias_halfwidth=0.05, gate_up_std=0.05,
                        down_std=0.05)


def test_ragged_bf16_tiles():
    """d and I not multiples of the 256/128 tile widths; N not a tile multiple."""
    m, x, layer, out, r = run(SMALL_BF16)
    full_check(SMALL_BF16, x, layer, out, r)


def test_all_experts_selected():
    w = SMALL_BF16.scaled(n_experts=4, top_k=4, d=128, d_ff=128, n_tokens=50)
    m, x, layer, out, r = run(w)
    full_check(w, x, layer, out, r)


def test_one_expert_takes_every_token():
    """k = 1 with a dominant bias: one expert gets 1000 rows (8 row tiles), the
    other experts stay empty."""
    w = SMALL_BF16.scaled(n_experts=8, top_k=1, d=256, d_ff=256, n_tokens=1000)
    layer = W.make_layer(w, 0, DEV)
    layer["bias"] = torch.zeros_like(layer["bias"])
    layer["bias"][3] = 5.0
    m, x, layer, out, r = run(w, layer=layer)
    res = full_check(w, x, layer, out, r)
    assert res["counts"][3] == 1000 and res["counts"].sum() == 1000


@pytest.mark.parametrize("n", [1, 7, 64, 65, 129])
def test_small_batches_decode_shapes(n):
    w = W.DECODE.scaled(n_tokens=n)
    m, x, layer, out, r = run(w, max_tokens=256)
    full_check(w, x, layer, out, r)


def test_fp32_ragged():
    w = W.TINY_F32.scaled(n_tokens=77, d=100, d_ff=70, n_experts=12, top_k=3)
    m, x, layer, out, r = run(w)
    full_check(w, x, layer, out, r)


def test_deterministic_in_place_and_host_path():
    w = W.DECODE.scaled(n_tokens=64)
    layer = W.make_layer(w, 0, DEV)
    x = W.make_x(w, DEV)
    m = MoeLayer(layer, w.top_k, w.eps, max_tokens=64)
    a = m(x)
    b = m(x)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    xi = x.clone()
    m(xi, out=xi)
    torch.cuda.synchronize()
    assert torch.equal(xi, a)
    xh = x.cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    m.forward_host(xh, oh)  # pinned: the last kernel stores into it
    assert torch.equal(oh, a.cpu())
    op = torch.empty_like(x.cpu())
    m.forward_host(xh, op)  # pageable: a copy from device staging
    assert torch.equal(op, a.cpu())
    big = torch.empty(xh.numel() + 4, dtype=xh.dtype).pin_memory()
    om = big[4:].view_as(xh)  # pinned but 8 bytes off a 16-byte boundary: staging
    m.forward_host(xh, om)
    assert torch.equal(om, a.cpu())
    # pinned in and out: a captured graph, replayed while the buffers and the
    # batch size stay; it reads the buffers' current contents
    x2 = W.make_x(w, DEV, seed=w.seed + 1)
    a2 = m(x2)
    torch.cuda.synchronize()
    for xin, ref in ((x, a), (x2, a2), (x, a)):
        xh.copy_(xin.cpu())
        oh.zero_()
        m.forward_host(xh, oh)
        assert torch.equal(oh, ref.cpu())
    # another batch size into the same buffers: a new capture, then the old size again
    h16 = xh[:16]
    o16 = oh[:16]
    ref16 = m(x[:16].contiguous())
    torch.cuda.synchronize()
    m.forward_host(h16, o16)
    assert torch.equal(o16, ref16.cpu())
    m.forward_host(xh, oh)
    assert torch.equal(oh, a.cpu())
    assert m.status() == 0


def test_zero_tokens_and_limits():
    w = W.DECODE.scaled(n_tokens=16)
    layer = W.make_layer(w, 0, DEV)
    m = MoeLayer(layer, w.top_k, w.eps, max_tokens=16)
    x = W.make_x(w, DEV)
    empty = x[:0]
    m(empty, out=torch.empty_like(empty))
    big = W.make_x(w, DEV, n_tokens=17)
    with pytest.raises(MoeError) as ei:
        m(big)
    assert ei.value.code == -4
    raw = torch.empty(16 * 2048 * 2 + 8, dtype=torch.uint8, device=DEV)
    mis = raw[2:2 + 16 * 2048 * 2].view(torch.bfloat16).view(16, 2048)
    with pytest.raises(MoeError) as ei:
        m(mis)
    assert ei.value.code == -3
    torch.cuda.synchronize()
    assert m.status() == 0


def test_bounded_wait_reports_timeout():
    w = W.TINY_F32
    layer = W.make_layer(w, 0, DEV)
    m = MoeLayer(layer, w.top_k, w.eps, max_tokens=64)
    m.selftest_timeout(2000)
    assert m.status() == -7
    assert m.status() == 0
    out = m(W.make_x(w, DEV))
    torch.cuda.synchronize()
    assert m.status() == 0 and torch.isfinite(out).all()


def test_bad_shapes_rejected():
    layer = W.make_layer(SMALL_BF16, 0, DEV)
    bad = dict(layer)
    bad["w_gate_up"] = layer["w_gate_up"][:, :, :200].contiguous()   # d = 200, not % 64
    with pytest.raises(MoeError) as ei:
        MoeLayer(bad, 4, 1e-6)
    assert ei.value.code == -2
    with pytest.raises(MoeError) as ei:
        MoeLayer(layer, 17, 1e-6)                                    # k > E
    assert ei.value.code == -2


def test_fused_path_one_expert_many_passes():
    """Small batches use the fused expert kernel (mean load <= 32 rows per
    expert); one expert taking all 200 tokens makes it stream that expert's
    weights in four passes of at most 64 tokens."""
    w = W.DECODE.scaled(n_tokens=200, top_k=1)
    layer = W.make_layer(w, 0, DEV)
    layer["bias"] = torch.zeros_like(layer["bias"])
    layer["bias"][7] = 5.0
    m, x, layer, out, r = run(w, layer=layer)
    assert m.launches_per_forward(200) == 4
    res = full_check(w, x, layer, out, r)
    assert res["counts"][7] == 200


def test_fused_path_all_experts_selected_ragged():
    w = SMALL_BF16.scaled(n_experts=8, top_k=8, d=320, d_ff=192, n_tokens=16)
    m, x, layer, out, r = run(w)
    assert m.launches_per_forward(16) == 4
    full_check(w, x, layer, out, r)


def test_both_expert_paths_agree():
    """The same 32 tokens through the fused kernel (batch of 32) and through
    the row-tiled GEMMs (inside a batch of 1024) agree within bf16 rounding."""
    w = W.DECODE.scaled(n_tokens=1024)
    layer = W.make_layer(w, 0, DEV)
    x = W.make_x(w, DEV)
    big = MoeLayer(layer, w.top_k, w.eps, max_tokens=1024)
    small = MoeLayer(layer, w.top_k, w.eps, max_tokens=32)
    assert big.launches_per_forward(1024) == 5 and small.launches_per_forward(32) == 4
    o_big = big(x)[:32]
    o_small = small(x[:32].contiguous())
    torch.cuda.synchronize()
    rel = (o_big.float() - o_small.float()).norm(dim=1) / o_small.float().norm(dim=1)
    assert rel.max().item() < 1e-2


def test_fp32_large_batch_tiled_router():
    """A large fp32 batch (ragged N) goes through the d-split cluster router."""
    w = W.TINY_F32.scaled(n_tokens=4100)
    m, x, layer, out, r = run(w)
    full_check(w, x, layer, out, r, tokens="sample")


@pytest.mark.parametrize("pair", ["1", "0"])
def test_grouped_gemms_ragged(monkeypatch, pair):
    """The CTA-pair GEMMs (256 weight rows per pair tile) and the single-CTA
    GEMMs (128-token tiles) on ragged shapes: d and I not multiples of the
    tile widths, experts whose rows end in the leader's half of a pair tile,
    and empty experts."""
    monkeypatch.setenv("MOE_TC_PAIR", pair)
    m, x, layer, out, r = run(SMALL_BF16)
    full_check(SMALL_BF16, x, layer, out, r)
    w = SMALL_BF16.scaled(n_experts=8, top_k=1, d=256, d_ff=256, n_tokens=1000)
    layer = W.make_layer(w, 0, DEV)
    layer["bias"] = torch.zeros_like(layer["bias"])
    layer["bias"][3] = 5.0
    m, x, layer, out, r = run(w, layer=layer)
    res = full_check(w, x, layer, out, r)
    assert res["counts"][3] == 1000


def test_single_and_pair_gemms_agree(monkeypatch):
    """One batch of 4096 tokens through the single-CTA and the CTA-pair
    grouped GEMMs: the same routing, outputs equal within bf16 rounding."""
    w = W.PREFILL.scaled(n_tokens=4096)
    layer = W.make_layer(w, 0, DEV)
    x = W.make_x(w, DEV)
    outs = []
    for mode in ("0", "1"):
        monkeypatch.setenv("MOE_TC_PAIR", mode)
        m = MoeLayer(layer, w.top_k, w.eps, max_tokens=w.n_tokens)
        outs.append(m(x).float())
        torch.cuda.synchronize()
        assert m.status() == 0
        m.close()
    rel = (outs[0] - outs[1]).norm(dim=1) / outs[1].norm(dim=1)
    assert rel.max().item() < 1e-2


def test_tc_router_ragged_small(monkeypatch):
    """The tensor-core router (forced on) on a ragged batch: 300 tokens (two
    full 128-token tiles and a tail), d = 320, E = 16."""
    monkeypatch.setenv("MOE_ROUTE_TC", "1")
    m, x, layer, out, r = run(SMALL_BF16)
    full_check(SMALL_BF16, x, layer, out, r)


@pytest.mark.parametrize("n_experts,top_k,d,n", [(64, 8, 2048, 777), (80, 6, 128, 513),
                                                 (16, 1, 64, 129)])
def test_tc_router_shapes(monkeypatch, n_experts, top_k, d, n):
    """Expert counts 16..80 (3E = 48..240 MMA columns), top-k 1..8, d from 64,
    token counts off the tile size; with k = 8 the dispatch chunks hold 64
    tokens, so a 128-token tile adds to two chunks' histograms."""
    monkeypatch.setenv("MOE_ROUTE_TC", "1")
    w = SMALL_BF16.scaled(n_experts=n_experts, top_k=top_k, d=d, d_ff=128, n_tokens=n,
                          router_std=0.05)
    m, x, layer, out, r = run(w)
    full_check(w, x, layer, out, r, tokens="sample")


def test_tc_and_simt_routers_agree(monkeypatch):
    """The same 2048-token batch through both routers: identical expert sets
    and slot order away from near ties, weights within fp32 rounding."""
    w = W.PREFILL.scaled(n_tokens=2048)
    layer = W.make_layer(w, 0, DEV)
    x = W.make_x(w, DEV)
    res = []
    for mode in ("0", "1"):
        monkeypatch.setenv("MOE_ROUTE_TC", mode)
        m = MoeLayer(layer, w.top_k, w.eps, max_tokens=w.n_tokens)
        m(x)
        torch.cuda.synchronize()
        assert m.status() == 0
        r = m.debug_routing(w.n_tokens)
        res.append((r["idx"].cpu(), r["w"].cpu()))
        m.close()
    same = (res[0][0] == res[1][0]).all(dim=1)
    assert same.float().mean().item() > 0.999
    torch.testing.assert_close(res[0][1][same], res[1][1][same], rtol=1e-5, atol=1e-7)


@pytest.mark.parametrize("n_experts,top_k,n,pair", [(256, 8, 300, "1"), (128, 4, 64, "1"),
                                                    (256, 4, 4096, "1"), (256, 4, 4096, "0")])
def test_many_experts(monkeypatch, n_experts, top_k, n, pair):
    """Up to the largest expert count (256) and top-k (8): the SIMT routers'
    expert blocks, a 256-column dispatch histogram, the fused expert kernel
    (N*k <= 32*E), and both the CTA-pair and the single-CTA GEMMs
    (4096 tokens x 4 > 32 * 256, 16 rows per expert on average)."""
    monkeypatch.setenv("MOE_TC_PAIR", pair)
    w = SMALL_BF16.scaled(n_experts=n_experts, top_k=top_k, d=256, d_ff=128, n_tokens=n,
                          router_std=0.05)
    m, x, layer, out, r = run(w)
    full_check(w, x, layer, out, r, tokens="sample" if n > 512 else None)


@pytest.mark.parametrize("route_tc", ["0", "1"])
def test_wide_rows(monkeypatch, route_tc):
    """d = 8192 through the cluster router (its row slices near the shared-
    memory limit) and through the tensor-core router (128 K stages split over
    a cluster of four)."""
    monkeypatch.setenv("MOE_ROUTE_TC", route_tc)
    w = SMALL_BF16.scaled(n_experts=16, top_k=4, d=8192, d_ff=128, n_tokens=96)
    m, x, layer, out, r = run(w)
    full_check(w, x, layer, out, r)


def test_fp32_widest_rows():
    """The largest supported width, d = 32768, in fp32: the large router's
    d-chunked tiles, a 128 KB gain vector in the dispatch's shared memory,
    the SIMT expert GEMMs."""
    w = W.TINY_F32.scaled(n_tokens=20, d=32768, d_ff=16, n_experts=8, top_k=2,
                          router_std=1.0 / 181.0, gate_up_std=1.0 / 181.0, down_std=0.25)
    m, x, layer, out, r = run(w)
    full_check(w, x, layer, out, r)


# ---------------------------------------------------------------- FP8_BLOCK
# The FP8 checkpoint's experts ("LFM2.5-24B-A2B: ein 24B-Reasoning-Modell, das pro Wortstück so wenig verbraucht wie ein 2B-Modell",
# inferencekey.com, section "Für Engineers", paragraph "Quantisierung"):
# e4m3 weights in 128x128 blocks, activations
# quantised per group of 128 inside the forward.

def fp8_small(**kw):
    """Small FP8_BLOCK shapes with weights of std 1/sqrt(K), so that the MoE
    part of out is as large as the residual and its error is measurable."""
    d, I = kw["d"], kw["d_ff"]
    return W.DECODE_FP8.scaled(router_std=0.05, gate_up_std=d ** -0.5, down_std=I ** -0.5, **kw)


def test_fp8_decode_full():
    """The 32-token decode step with FP8_BLOCK experts, every token."""
    w = W.DECODE_FP8
    m, x, layer, out, r = run(w)
    assert m.launches_per_forward(w.n_tokens) == 4
    res = full_check(w, x, layer, out, r)
    assert (res["counts"] > 0).sum() >= 45


@pytest.mark.parametrize("n_experts,top_k,d,d_ff,n", [(8, 2, 256, 256, 100), (16, 4, 384, 640, 333),
                                                      (4, 4, 128, 128, 1)])
def test_fp8_ragged(n_experts, top_k, d, d_ff, n):
    """Ragged FP8_BLOCK shapes: passes of 64 tokens with ragged tails, several
    K blocks of both contractions, k = E, a single token."""
    w = fp8_small(n_experts=n_experts, top_k=top_k, d=d, d_ff=d_ff, n_tokens=n)
    m, x, layer, out, r = run(w)
    full_check(w, x, layer, out, r)


def test_fp8_one_expert_takes_all():
    """One expert receives all 700 tokens (11 passes of 64 per item, the
    others empty): the act rows of many passes before the down items."""
    w = fp8_small(n_experts=8, top_k=1, d=256, d_ff=384, n_tokens=700)
    layer = W.make_layer(w, 0, DEV)
    layer["bias"] = torch.zeros_like(layer["bias"])
    layer["bias"][5] = 5.0
    m, x, layer, out, r = run(w, layer=layer)
    res = full_check(w, x, layer, out, r)
    assert res["counts"][5] == 700


def test_fp8_many_passes_in_the_small_batch_shape():
    """200 tokens, k = 1, all on one of 8 experts: still the 32-token shape
    (N*k <= 32*E), so that expert's items run in 7 passes, which must all be
    published before its down items read the act rows."""
    w = fp8_small(n_experts=8, top_k=1, d=256, d_ff=256, n_tokens=200)
    layer = W.make_layer(w, 0, DEV)
    layer["bias"] = torch.zeros_like(layer["bias"])
    layer["bias"][2] = 5.0
    m, x, layer, out, r = run(w, layer=layer)
    res = full_check(w, x, layer, out, r)
    assert res["counts"][2] == 200


def test_fp8_quantised_rows_match_the_oracle():
    """The dispatch's e4m3 rows: each grouped row holds the codes and group
    scales of its token's normalised row (oracle RMSNorm, quantised by the
    oracle). Scales agree to fp32 rounding; a code may differ only by one
    step, where v / s lies within a hair of a rounding midpoint."""
    import oracle
    w = W.DECODE_FP8.scaled(n_tokens=96)
    m, x, layer, out, r = run(w)
    q = m.debug_fp8_rows(w.n_tokens)
    torch.cuda.synchronize()
    perm = r["perm"].cpu().numpy()
    tok = perm // w.top_k
    xn = oracle.rmsnorm(x.cpu(), layer["norm_gain"].cpu(), w.eps)
    ref = oracle.quant(xn[tok])
    np.testing.assert_allclose(q["scales"].cpu().numpy(), ref["scales"], rtol=2e-6)
    codes = q["codes"].cpu().numpy()
    same = codes == ref["codes"]
    assert same.mean() > 0.999, same.mean()
    vals_g = oracle.e4m3_value(codes[~same])
    vals_r = oracle.e4m3_value(ref["codes"][~same])
    s = np.repeat(ref["scales"], 128, axis=1)[~same]
    v = xn[tok][~same] / s
    # both neighbours of v: the two codes bracket v and v sits near their midpoint
    assert np.all(np.minimum(vals_g, vals_r) <= v + 1e-6 * np.abs(v)), "code not adjacent"
    assert np.all(np.maximum(vals_g, vals_r) >= v - 1e-6 * np.abs(v)), "code not adjacent"
    mid = (vals_g + vals_r) / 2
    assert np.all(np.abs(v - mid) <= 1e-5 * np.abs(v) + 1e-12), "flip away from a midpoint"


def test_fp8_prefill_sampled():
    """8192 tokens with FP8_BLOCK experts (about 512 rows per expert: eight
    passes per weight tile) on sampled tokens."""
    w = W.PREFILL_FP8
    m, x, layer, out, r = run(w)
    full_check(w, x, layer, out, r, tokens="sample")


def test_fp8_deterministic_and_in_place():
    w = W.DECODE_FP8.scaled(n_tokens=200)
    layer = W.make_layer(w, 0, DEV)
    x = W.make_x(w, DEV)
    m = MoeLayer(layer, w.top_k, w.eps, max_tokens=w.n_tokens)
    a = m(x)
    b = m(x)
    xi = x.clone()
    m(xi, out=xi)
    torch.cuda.synchronize()
    assert m.status() == 0
    assert torch.equal(a, b) and torch.equal(a, xi)


def _fp8_layer_pair(w, layer, pair_mode):
    """A context over the layer with the CTA-pair FP8 GEMMs on (default) or
    off (MOE_FP8_PAIR=0: the persistent FP8 kernel for every batch)."""
    import os
    old = os.environ.pop("MOE_FP8_PAIR", None)
    try:
        if pair_mode == 0:
            os.environ["MOE_FP8_PAIR"] = "0"
        return MoeLayer(layer, w.top_k, w.eps, w.routed_scale, max_tokens=w.n_tokens)
    finally:
        os.environ.pop("MOE_FP8_PAIR", None)
        if old is not None:
            os.environ["MOE_FP8_PAIR"] = old


@pytest.mark.parametrize("shape", [dict(n_experts=16, top_k=4, d=384, d_ff=640, n_tokens=700),
                                   dict(n_experts=64, top_k=4, d=2048, d_ff=1536, n_tokens=2048)])
def test_fp8_pair_and_persistent_kernels_agree(shape):
    """Large FP8_BLOCK batches through the CTA-pair GEMMs and through the
    persistent kernel: the same e4m3 products, per-K-block promotion with the
    same factors, the same SiLU and quantisation, so the outputs agree to the
    bf16 rounding of y and out (measured: most rows bit-identical)."""
    w = fp8_small(**shape)
    layer = W.make_layer(w, 0, DEV)
    x = W.make_x(w, DEV)
    a = _fp8_layer_pair(w, layer, -1)
    b = _fp8_layer_pair(w, layer, 0)
    assert a.launches_per_forward(w.n_tokens) == 6 and b.launches_per_forward(w.n_tokens) == 4
    oa, ob = a(x), b(x)
    torch.cuda.synchronize()
    assert a.status() == 0 and b.status() == 0
    ra, rb = a.debug_routing(w.n_tokens), b.debug_routing(w.n_tokens)
    assert torch.equal(ra["idx"], rb["idx"]) and torch.equal(ra["perm"], rb["perm"])
    da, db = (oa.double() - x.double()), (ob.double() - x.double())
    rel = (da - db).norm(dim=1) / da.norm(dim=1).clamp_min(1e-30)
    assert rel.max().item() <= 2e-2, rel.max().item()
    a.close()
    b.close()


def test_fp8_large_batch_deterministic_and_in_place():
    w = W.DECODE_FP8.scaled(n_tokens=1500)
    layer = W.make_layer(w, 0, DEV)
    x = W.make_x(w, DEV)
    m = MoeLayer(layer, w.top_k, w.eps, max_tokens=w.n_tokens)
    assert m.launches_per_forward(w.n_tokens) == 6
    m.profile(True)
    a = m(x)
    assert list(m.kernel_times()) == ["route", "dispatch", "gate_up", "quantize", "down", "combine"]
    m.profile(False)
    b = m(x)
    xi = x.clone()
    m(xi, out=xi)
    torch.cuda.synchronize()
    assert m.status() == 0
    assert torch.equal(a, b) and torch.equal(a, xi)
    m.close()


def test_fp8_quantiser_division_is_the_ieee_quotient():
    """The FP8 quantisers divide by a scale through its reciprocal and one
    correction step; the quotient must equal the IEEE one bit for bit
    wherever it is a normal float (the codes are e4m3 of it)."""
    from sigmoid_bias_top_b200 import selftest_fp8_divide
    g = torch.Generator().manual_seed(7)
    n = 1 << 22
    a = torch.randn(n, generator=g) * torch.exp2(torch.randint(-20, 21, (n,), generator=g).float())
    # divisors as the quantisers meet them: amax / 448 over a wide range,
    # plus significands with every bit set and exact powers of two
    b = (torch.rand(n, generator=g) + 0.5) * torch.exp2(torch.randint(-40, 30, (n,), generator=g).float())
    b[: n // 8] = torch.exp2(torch.randint(-40, 30, (n // 8,), generator=g).float())
    ones = torch.tensor([float.fromhex("0x1.fffffep0")])
    b[n // 8: n // 4] = ones * torch.exp2(torch.randint(-40, 30, (n // 8,), generator=g).float())
    # numerators whose quotient lies next to a rounding midpoint
    m = torch.randint(1 << 23, 1 << 24, (n // 8,), generator=g).double() + 0.5
    a[n // 4: 3 * n // 8] = (m * b[n // 4: 3 * n // 8].double() * 2.0 ** -23).float()
    a[:16] = 0.0
    a[16:32] = -a[16:32]
    b[32:48] = 2.0 ** -110      # outside the reciprocal's safe range:
    b[48:64] = 2.0 ** 110       # the full division
    b = b.to(DEV)
    q, q_ref = selftest_fp8_divide(a.to(DEV), b)
    torch.cuda.synchronize()
    normal = q_ref.abs() >= 2.0 ** -126
    assert torch.equal(q[normal].view(torch.int32), q_ref[normal].view(torch.int32))
    assert torch.equal(q[q_ref == 0], q_ref[q_ref == 0])
    # below the normal range both are tiny; e4m3 of either is code 0
    assert (q[~normal & (q_ref != 0)].abs() < 2.0 ** -120).all()
