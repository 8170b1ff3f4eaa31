"""Algorithmic work of one MoE-block forward: the byte and FLOP counts that
throughput and roofline fractions are computed from.

Counts follow "LFM2.5-24B-A2B: Biased Routing, Short Convolutions and Ten KV
Caches" (flozi.net, English page): section "The router has two different
scores" (an expert is three matrices, 3 x 2048 x 1536 = 9,437,184 weights) and
section "Active weights do not define resident memory" (a multiply-add counts
as two FLOPs; the selected experts cost 2 x 38 x 4 x 3 x 2048 x 1536 FLOPs per
token over 38 MoE layers).
"""
from __future__ import annotations


def expert_weights(d: int, d_ff: int) -> int:
    """Weights of one gated-SiLU expert: gate, up and down matrices."""
    return 3 * d * d_ff


def expert_flops_per_token(d: int, d_ff: int, top_k: int, n_layers: int = 1) -> int:
    """Selected-expert matrix FLOPs per token (multiply-add = 2)."""
    return 2 * n_layers * top_k * expert_weights(d, d_ff)


def router_flops_per_token(d: int, n_experts: int) -> int:
    return 2 * d * n_experts


def decode_bytes(active_experts: int, n_tokens: int, d: int, d_ff: int, n_experts: int,
                 w_bytes: int = 2, x_bytes: int = 2) -> int:
    """HBM bytes a weight-streaming forward must move: the active experts'
    weights, the fp32 router matrix, gain and bias, x read and out written.
    Intermediates and unselected experts are not counted."""
    return (active_experts * expert_weights(d, d_ff) * w_bytes
            + n_experts * d * 4 + d * 4 + n_experts * 4
            + 2 * n_tokens * d * x_bytes)


def gate_up_bytes(active_experts: int, d: int, d_ff: int, w_bytes: int = 2) -> int:
    """Weight bytes the packed gate/up grouped GEMM must stream."""
    return active_experts * 2 * d_ff * d * w_bytes


def down_bytes(active_experts: int, d: int, d_ff: int, w_bytes: int = 2) -> int:
    return active_experts * d * d_ff * w_bytes


def gate_up_flops(n_assign: int, d: int, d_ff: int) -> int:
    """Tensor FLOPs of the gate/up contraction over all token-expert pairs."""
    return 2 * n_assign * 2 * d_ff * d


def down_flops(n_assign: int, d: int, d_ff: int) -> int:
    return 2 * n_assign * d * d_ff


# FP8_BLOCK experts ("LFM2.5-24B-A2B: ein 24B-Reasoning-Modell, das pro Wortstück so wenig verbraucht wie ein 2B-Modell",
# inferencekey.com, section "Für Engineers", paragraph "Quantisierung":
# weights FP8 in static 128x128 blocks, activations FP8 per group of 128).

def fp8_scale_bytes(active_experts: int, d: int, d_ff: int) -> int:
    """fp32 block scales of the active experts' gate/up and down matrices."""
    blocks = (-(-2 * d_ff // 128)) * (-(-d // 128)) + (-(-d // 128)) * (-(-d_ff // 128))
    return active_experts * blocks * 4


def fp8_experts_bytes(active_experts: int, n_assign: int, d: int, d_ff: int) -> int:
    """Bytes the FP8 expert kernel (both contractions in one launch) must
    move: e4m3 weights (1 byte each) and their block scales; the grouped e4m3
    input rows and their group scales read; SiLU(gate)*up codes and scales
    written and read back; the bf16 expert outputs written."""
    rows_in = n_assign * (d + 4 * (-(-d // 128)))
    act = 2 * n_assign * (d_ff + 4 * (-(-d_ff // 128)))
    return (active_experts * expert_weights(d, d_ff) + fp8_scale_bytes(active_experts, d, d_ff)
            + rows_in + act + n_assign * d * 2)


# Neighbouring steps of the block ("LFM2.5-24B-A2B: Biased Routing, Short
# Convolutions and Ten KV Caches", sections "The exact checkpoint" and "A
# short convolution is a local mixer, not an embedding lookup"): per launch
# of each kernel, the tensor FLOPs (multiply-add = 2) and the bytes it must
# move at least (weights once, its input rows read, its output rows written;
# bf16 = 2 bytes).

def block_kernel_work(kind: str, kernel: str, n: int, d: int, d_ff: int = 0):
    """(flops, bytes) of one launch of a dense / conv block kernel over n tokens."""
    b = 2
    if kind == "dense":
        I = d_ff
        table = {
            "norm": (0, 2 * n * d * b),
            "gate_up": (2 * n * 2 * I * d, 2 * I * d * b + n * d * b + n * I * b),
            "down_residual": (2 * n * d * I, d * I * b + n * I * b + 2 * n * d * b),
            # split-K (small batches): the GEMMs' fp32 partial sums are
            # intermediates; the reduce launches write the step's output
            "gate_up_split": (2 * n * 2 * I * d, 2 * I * d * b + n * d * b),
            "gate_up_reduce": (0, n * I * b),
            "down_split": (2 * n * d * I, d * I * b + n * I * b),
            "down_residual_reduce": (0, 2 * n * d * b),
        }
    else:
        table = {
            "norm": (0, 2 * n * d * b),
            "in_gv": (2 * n * 2 * d * d, 2 * d * d * b + n * d * b + n * d * b),
            "in_u_conv": (2 * n * d * d, d * d * b + n * d * b + n * d * b + n * d * b),
            "out_residual": (2 * n * d * d, d * d * b + n * d * b + 2 * n * d * b),
            "state": (0, 0),
            "in_gv_split": (2 * n * 2 * d * d, 2 * d * d * b + n * d * b),
            "in_gv_reduce": (0, n * d * b),
            "in_u_split": (2 * n * d * d, d * d * b + n * d * b),
            "in_u_conv_reduce": (0, 2 * n * d * b),
            "out_split": (2 * n * d * d, d * d * b + n * d * b),
            "out_residual_reduce": (0, 2 * n * d * b),
        }
    return table[kernel]


def block_flops_per_token(kind: str, d: int, d_ff: int = 0) -> int:
    """Tensor FLOPs per token of a whole dense or conv block."""
    return 2 * 3 * d * d_ff if kind == "dense" else 2 * 4 * d * d
