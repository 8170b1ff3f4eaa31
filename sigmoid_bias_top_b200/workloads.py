"""Seeded synthetic inputs for the sigmoid-bias top-k MoE feed-forward block.

This module only draws random tensors of the shapes and distributions of the
workloads; it contains none of the layer's arithmetic (no norm, no
routing, no expert math), so that the CUDA path and the CPU oracle can both be
fed from it without sharing any computation.

Shapes follow "LFM2.5-24B-A2B: Biased Routing, Short Convolutions and Ten KV
Caches" (flozi.net, English page), section "The router has two different
scores": hidden width 2048, 64 experts, top-4, expert intermediate 1536, a
fp32 router matrix W_r[E x d] and a stored 64-element expert bias.

Tensor layout (what the C ABI consumes):
  x          [N, d]        f32 or bf16   residual stream (the block input)
  norm_gain  [d]           f32           RMSNorm gain, multiplied as stored
  router_w   [E, d]        f32           router matrix, row-major
  bias       [E]           f32           expert bias (selection only)
  w_gate_up  [E, 2I, d]    f32 or bf16   rows 0..I-1 = gate, rows I..2I-1 = up
  w_down     [E, d, I]     f32 or bf16   down projection
FP8_BLOCK workloads (dtype "fp8"; the FP8 checkpoint of "LFM2.5-24B-A2B: ein 24B-Reasoning-Modell, das pro Wortstück so wenig verbraucht wie ein 2B-Modell",
inferencekey.com, section "Für Engineers", paragraphs "Checkpoint" and
"Quantisierung") keep x bf16 and store the expert
matrices as e4m3 codes (torch.float8_e4m3fn) with fp32 block scales:
  w_gate_up_scale [E, 2I/128, d/128]   w_down_scale [E, d/128, I/128]
The codes are normal draws of standard deviation fp8_code_std cast to e4m3
(saturating at 448) and every block scale is std / fp8_code_std times a
uniform factor in (0.9, 1.1), so that code * scale has the std of the bf16
workloads' weights; for N(0, std) blocks of 128 x 128 values a static
amax / 448 scale would put the codes at about this spread.
Distribution parameters written "N(0, v)" with v a fraction of the width
(1/256, 1/192) are variances; "N(0, 0.02)" is a standard deviation, the usual
initializer-range convention.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Dict, List, Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    n_tokens: int
    d: int
    n_experts: int
    top_k: int
    d_ff: int
    dtype: str                      # "f32", "bf16" (x, out, experts) or "fp8" (bf16 x)
    eps: float = 1e-6
    routed_scale: float = 1.0
    n_layers: int = 1
    seed: int = 0
    x_std: float = 1.0
    gain_jitter: float = 0.0        # gain = 1 + N(0, jitter^2)
    router_std: float = 0.02
    bias_kind: str = "uniform"      # "uniform", "zero", "zipf"
    bias_halfwidth: float = 0.05    # uniform bias in (-h, h)
    gate_up_std: float = 0.02
    down_std: float = 0.02
    # skewed-load bias: b_e = zipf_scale * log p_rank(e) - zipf_tail_drop on the
    # zipf_tail lowest ranks, with p_r proportional to r^-zipf_s
    zipf_s: float = 1.2
    zipf_scale: float = 0.08
    zipf_tail: int = 4
    zipf_tail_drop: float = 0.15
    fp8_code_std: float = 109.0

    @property
    def torch_dtype(self) -> torch.dtype:
        """Storage type of x and out."""
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


TINY_F32 = Workload(
    name="tiny_f32_N64_d256_E16_k4_I192", n_tokens=64, d=256, n_experts=16, top_k=4,
    d_ff=192, dtype="f32", seed=1, x_std=1.0, gain_jitter=0.0,
    router_std=1.0 / 16.0, bias_kind="uniform", bias_halfwidth=0.5,
    gate_up_std=1.0 / 16.0, down_std=1.0 / math.sqrt(192.0))

DECODE = Workload(
    name="decode_N32_d2048_E64_k4_I1536", n_tokens=32, d=2048, n_experts=64, top_k=4,
    d_ff=1536, dtype="bf16", seed=2, gain_jitter=0.02, router_std=0.02,
    bias_kind="uniform", bias_halfwidth=0.05)

PREFILL = Workload(
    name="prefill_N8192_d2048_E64_k4_I1536", n_tokens=8192, d=2048, n_experts=64,
    top_k=4, d_ff=1536, dtype="bf16", seed=3, gain_jitter=0.02, router_std=0.02,
    bias_kind="zero")

SKEWED = Workload(
    name="skewed_prefill_N16384_d2048_E64_k4_I1536", n_tokens=16384, d=2048,
    n_experts=64, top_k=4, d_ff=1536, dtype="bf16", seed=4, gain_jitter=0.02,
    router_std=0.02, bias_kind="zipf")

STACKED = Workload(
    name="stacked_decode_L38_N256_d2048_E64_k4_I1536", n_tokens=256, d=2048,
    n_experts=64, top_k=4, d_ff=1536, dtype="bf16", seed=5, n_layers=38,
    gain_jitter=0.02, router_std=0.02, bias_kind="uniform", bias_halfwidth=0.05)

# Speculative-decoding verify step: the drafter of "LFM2.5-24B-A2B-DSpark ist
# live auf Hugging Face" (orcarouter.ai, section "Was ist eigentlich im
# Repository?") proposes blocks of 9 tokens, so the target verifies 9 + 1
# tokens per sequence at once; 32 sequences give 320 tokens per step, whose
# expert union is wider than a 32-token decode step's (section "Die fehlende
# Mac-Nummer ist die interessante Auslassung.").
VERIFY = Workload(
    name="verify_B32x10_N320_d2048_E64_k4_I1536", n_tokens=320, d=2048, n_experts=64,
    top_k=4, d_ff=1536, dtype="bf16", seed=6, gain_jitter=0.02, router_std=0.02,
    bias_kind="uniform", bias_halfwidth=0.05)

# The decode and prefill steps with the FP8 checkpoint's FP8_BLOCK experts.
DECODE_FP8 = DECODE.scaled(name="decode_fp8_N32_d2048_E64_k4_I1536", dtype="fp8", seed=7)
PREFILL_FP8 = PREFILL.scaled(name="prefill_fp8_N8192_d2048_E64_k4_I1536", dtype="fp8", seed=8)

WORKLOADS: Dict[str, Workload] = {
    "tiny": TINY_F32, "decode": DECODE, "prefill": PREFILL, "skewed": SKEWED,
    "stacked": STACKED, "verify": VERIFY, "decode_fp8": DECODE_FP8,
    "prefill_fp8": PREFILL_FP8,
}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal(shape, std, g, device, dtype):
    # drawn in f32 then stored in the target dtype; the stored values are the truth
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(dtype)


def zipf_bias(w: Workload, g: torch.Generator, device) -> torch.Tensor:
    """Expert bias for the skewed-load workload: a log-Zipf profile over ranks,
    ranks assigned to experts by a seeded permutation."""
    E = w.n_experts
    r = torch.arange(1, E + 1, dtype=torch.float64)
    p = r.pow(-w.zipf_s)
    p = p / p.sum()
    b_rank = w.zipf_scale * torch.log(p)
    b_rank[E - w.zipf_tail:] -= w.zipf_tail_drop
    perm = torch.randperm(E, generator=g, device=device).cpu()
    b = torch.empty(E, dtype=torch.float64)
    b[perm] = b_rank            # expert perm[r] gets rank r
    return b.to(torch.float32).to(device)


def make_layer(w: Workload, layer: int = 0, device="cpu",
               seed: Optional[int] = None, with_experts: bool = True) -> Dict[str, torch.Tensor]:
    """Weights of one MoE block (layer index selects an independent stream).

    with_experts=False stops after the router tensors (same values as a full
    draw, since the expert matrices are drawn last)."""
    base = w.seed if seed is None else seed
    g = _gen(device, 1_000_003 * (base + 1) + 7919 * (layer + 1))
    E, d, I = w.n_experts, w.d, w.d_ff
    dt = w.torch_dtype
    gain = torch.ones(d, device=device, dtype=torch.float32)
    if w.gain_jitter:
        gain = gain + _normal((d,), w.gain_jitter, g, device, torch.float32)
    router_w = _normal((E, d), w.router_std, g, device, torch.float32)
    if w.bias_kind == "uniform":
        bias = ((torch.rand(E, generator=g, device=device, dtype=torch.float32) * 2 - 1)
                * w.bias_halfwidth)
    elif w.bias_kind == "zero":
        bias = torch.zeros(E, device=device, dtype=torch.float32)
    elif w.bias_kind == "zipf":
        bias = zipf_bias(w, g, device)
    else:
        raise ValueError(w.bias_kind)
    out = {"norm_gain": gain.contiguous(), "router_w": router_w.contiguous(),
           "bias": bias.contiguous()}
    if with_experts and w.dtype == "fp8":
        cs = w.fp8_code_std
        for name, shape, std in (("w_gate_up", (E, 2 * I, d), w.gate_up_std),
                                 ("w_down", (E, d, I), w.down_std)):
            codes = (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * cs)
            out[name] = codes.clamp_(-448.0, 448.0).to(torch.float8_e4m3fn).contiguous()
            del codes
            blocks = (E, -(-shape[1] // 128), -(-shape[2] // 128))
            out[name + "_scale"] = ((0.9 + 0.2 * torch.rand(blocks, generator=g, device=device,
                                                             dtype=torch.float32))
                                    * (std / cs)).contiguous()
    elif with_experts:
        out["w_gate_up"] = _normal((E, 2 * I, d), w.gate_up_std, g, device, dt).contiguous()
        out["w_down"] = _normal((E, d, I), w.down_std, g, device, dt).contiguous()
    return out


def make_x(w: Workload, device="cpu", seed: Optional[int] = None,
           n_tokens: Optional[int] = None) -> torch.Tensor:
    base = w.seed if seed is None else seed
    g = _gen(device, 7 * (base + 1) + 3)
    n = w.n_tokens if n_tokens is None else n_tokens
    return _normal((n, w.d), w.x_std, g, device, w.torch_dtype).contiguous()


def make_inputs(w: Workload, device="cpu", seed: Optional[int] = None):
    """x plus the weights of every layer of the workload."""
    layers = [make_layer(w, l, device, seed) for l in range(w.n_layers)]
    return make_x(w, device, seed), layers


# ---------------------------------------------------------------------------
# The neighbouring steps of the block: dense feed-forward (layers 0-1) and the
# short-convolution mixer ("LFM2.5-24B-A2B: Biased Routing, Short
# Convolutions and Ten KV Caches", sections "The exact checkpoint" and "A
# short convolution is a local mixer, not an embedding lookup"). The page
# gives the width (2048) but not the dense intermediate width; 6144 = 3 x
# 2048 is the dense SwiGLU width the family's drafter uses at hidden 2048
# ("LFM2.5-24B-A2B-DSpark ist live auf Hugging Face", orcarouter.ai), taken
# here as the workload's. Tensors:
#   dense: norm_gain [d] f32, w_gate_up [2I, d], w_down [d, I] bf16
#   conv:  norm_gain [d] f32, w_in [3d, d] (g, u, v rows), w_out [d, d] bf16,
#          conv [d, 3] f32 taps by lag; x [B, T, d] bf16; state [B, 2, d] f32

@dataclass(frozen=True)
class BlockWorkload:
    name: str
    kind: str                  # "dense" or "conv"
    n_seqs: int                # B
    seq_len: int               # T
    d: int
    d_ff: int = 0              # dense intermediate width
    seed: int = 0
    eps: float = 1e-6
    x_std: float = 1.0
    gain_jitter: float = 0.02
    w_std: float = 0.02        # projection weights N(0, w_std^2)
    conv_std: float = 0.5      # taps N(0, conv_std^2)
    state_std: float = 0.8     # carried a vectors N(0, state_std^2) (decode)
    with_state: bool = False   # decode steps continue sequences with a carried state

    @property
    def n_tokens(self) -> int:
        return self.n_seqs * self.seq_len

    def scaled(self, **kw) -> "BlockWorkload":
        return replace(self, **kw)


DENSE_PREFILL = BlockWorkload("dense_prefill_B4xT2048_d2048_I6144", "dense", 4, 2048, 2048, 6144,
                              seed=21)
DENSE_DECODE = BlockWorkload("dense_decode_B32_d2048_I6144", "dense", 32, 1, 2048, 6144, seed=22)
CONV_PREFILL = BlockWorkload("conv_prefill_B4xT2048_d2048", "conv", 4, 2048, 2048, seed=23)
CONV_DECODE = BlockWorkload("conv_decode_B32_d2048", "conv", 32, 1, 2048, seed=24,
                            with_state=True)

BLOCK_WORKLOADS: Dict[str, BlockWorkload] = {
    "dense_prefill": DENSE_PREFILL, "dense_decode": DENSE_DECODE,
    "conv_prefill": CONV_PREFILL, "conv_decode": CONV_DECODE,
}


def make_block_layer(w: BlockWorkload, device="cpu", layer: int = 0) -> Dict[str, torch.Tensor]:
    g = _gen(device, 1_000_003 * (w.seed + 1) + 7919 * (layer + 1))
    d = w.d
    gain = torch.ones(d, device=device, dtype=torch.float32)
    if w.gain_jitter:
        gain = gain + _normal((d,), w.gain_jitter, g, device, torch.float32)
    out = {"norm_gain": gain.contiguous()}
    if w.kind == "dense":
        out["w_gate_up"] = _normal((2 * w.d_ff, d), w.w_std, g, device, torch.bfloat16).contiguous()
        out["w_down"] = _normal((d, w.d_ff), w.w_std, g, device, torch.bfloat16).contiguous()
    else:
        out["w_in"] = _normal((3 * d, d), w.w_std, g, device, torch.bfloat16).contiguous()
        out["conv"] = _normal((d, 3), w.conv_std, g, device, torch.float32).contiguous()
        out["w_out"] = _normal((d, d), w.w_std, g, device, torch.bfloat16).contiguous()
    return out


def make_block_x(w: BlockWorkload, device="cpu", seed: Optional[int] = None) -> torch.Tensor:
    """x: [N, d] for the dense block, [B, T, d] for the conv block (bf16)."""
    base = w.seed if seed is None else seed
    g = _gen(device, 7 * (base + 1) + 5)
    shape = (w.n_tokens, w.d) if w.kind == "dense" else (w.n_seqs, w.seq_len, w.d)
    return _normal(shape, w.x_std, g, device, torch.bfloat16).contiguous()


def make_conv_state(w: BlockWorkload, device="cpu", seed: Optional[int] = None) -> torch.Tensor:
    """A carried state [B, 2, d] f32 (the a vectors of two earlier positions)."""
    base = w.seed if seed is None else seed
    g = _gen(device, 11 * (base + 1) + 1)
    return _normal((w.n_seqs, 2, w.d), w.state_std, g, device, torch.float32).contiguous()
