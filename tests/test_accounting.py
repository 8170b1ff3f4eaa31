"""Shape and FLOP accounting against the numbers the page prints."""
from sigmoid_bias_top_b200 import accounting as A


def test_expert_weights_per_expert():
    # section "The router has two different scores": 3 x 2048 x 1536 = 9,437,184
    assert A.expert_weights(2048, 1536) == 9_437_184


def test_expert_parameter_totals():
    # section "Active weights do not define resident memory": experts hold about
    # 22.951 B over 38 layers; keeping 4 of 64 experts gives about 2.455 B active
    # out of 23,971,585,280 total.
    total_expert = 38 * 64 * A.expert_weights(2048, 1536)
    assert total_expert == 22_951_231_488
    assert round(total_expert / 1e9, 3) == 22.951
    active = 23_971_585_280 - 38 * 60 * A.expert_weights(2048, 1536)
    assert active == 2_454_805_760
    assert round(active / 1e9, 3) == 2.455


def test_expert_flops_per_token():
    # 2 x 38 x 4 x 3 x 2048 x 1536 ~ 2.869 GFLOP per token
    f = A.expert_flops_per_token(2048, 1536, top_k=4, n_layers=38)
    assert f == 2_868_903_936
    assert round(f / 1e9, 3) == 2.869
    # all 64 experts would cost 16 times as much for that term
    assert A.expert_flops_per_token(2048, 1536, 64, 38) == 16 * f


def test_split_counts_add_up():
    n = 8192 * 4
    assert A.gate_up_flops(n, 2048, 1536) + A.down_flops(n, 2048, 1536) == \
        8192 * A.expert_flops_per_token(2048, 1536, 4)
    assert A.gate_up_bytes(56, 2048, 1536) + A.down_bytes(56, 2048, 1536) == \
        56 * A.expert_weights(2048, 1536) * 2


def test_fp8_bytes():
    """One byte per e4m3 weight plus one fp32 scale per 128x128 block: the
    2048 x 1536 expert has 24 x 16 gate/up blocks and 16 x 12 down blocks."""
    assert A.fp8_scale_bytes(1, 2048, 1536) == (24 * 16 + 16 * 12) * 4
    w = A.fp8_experts_bytes(56, 0, 2048, 1536)
    assert w == 56 * (A.expert_weights(2048, 1536) + 2304)
    assert A.fp8_experts_bytes(56, 128, 2048, 1536) - w == \
        128 * (2048 + 64) + 2 * 128 * (1536 + 48) + 128 * 2048 * 2


def test_block_work_sums_to_the_block_flops():
    """The per-kernel FLOPs of the dense and conv blocks add up to the
    block's per-token count (dense: three d x I matrices; conv: W_in's three
    d x d streams and W_out), times the tokens."""
    n, d, I = 8192, 2048, 6144
    dense = sum(A.block_kernel_work("dense", k, n, d, I)[0]
                for k in ("norm", "gate_up", "down_residual"))
    conv = sum(A.block_kernel_work("conv", k, n, d)[0]
               for k in ("norm", "in_gv", "in_u_conv", "out_residual", "state"))
    assert dense == n * A.block_flops_per_token("dense", d, I) == 2 * n * 3 * d * I
    assert conv == n * A.block_flops_per_token("conv", d) == 2 * n * 4 * d * d


def test_bench_takes_the_burst_peak_unless_power_capped_or_long():
    import bench
    from sigmoid_bias_top_b200 import workloads as W
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    w = W.PREFILL
    ms = {"gate_up": 0.35}
    calm = {"reasons": []}
    capped = {"reasons": ["sw_power_cap"]}
    b = bench.roofline(w, "gate_up", ms, 64, peaks, "measured", calm, 0.2)
    assert b[0] == "tensor" and b[3] == 1600.0
    assert bench.roofline(w, "gate_up", ms, 64, peaks, "measured", capped, 0.2)[3] == 1400.0
    assert bench.roofline(w, "gate_up", ms, 64, peaks, "measured", calm, 1.5)[3] == 1400.0
    fp8 = bench.roofline(W.PREFILL_FP8, "experts", {"experts": 1.0}, 64, peaks, "measured",
                         calm, 0.2)
    assert fp8[3] == 3200.0                       # e4m3: twice the bf16 peak
    dec = bench.roofline(W.DECODE, "experts", {"experts": 0.17}, 54, peaks, "measured", calm, 0.1)
    assert dec[0] == "hbm" and dec[3] == 6000.0
