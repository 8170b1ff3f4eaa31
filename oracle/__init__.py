"""fp64 CPU oracle of the sigmoid-bias top-k MoE block (test infrastructure).

Only the tests, the package's smoke check and the benchmark's CPU-baseline leg
may import this package. The CUDA product path never imports it and shares no
code with it; it only shares the seeded input generator.

The arithmetic lives in moe_oracle.c (plain loops, double precision); this
module marshals torch/numpy CPU arrays into it. See the C file's header for the
passages each step follows.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from ._build import build

F32, BF16, F64, E4M3 = 0, 1, 2, 3

MUTATIONS = {
    "none": 0, "biased_weights": 1, "softmax": 2, "bias_before_act": 3,
    "no_eps": 4, "no_gain": 5, "silu_on_up": 6, "tie_high": 7,
    "no_residual": 8, "mean_not_sum": 9, "slot_swap": 10, "down_transposed": 11,
    "fp8_scale_transposed": 12, "fp8_no_act_quant": 13, "fp8_no_max": 14,
    "margin_zero": 15, "margin_worst_unselected": 16, "margin_on_s": 17,
    "forced_ignored": 18, "forced_weights_own_choice": 19,
    "conv_lag_reversed": 20, "conv_centered": 21, "conv_gate_after": 22,
    "conv_sequence_leak": 23, "conv_uv_swapped": 24,
}

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = build()
        L = ctypes.CDLL(path)
        P, I, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        L.oracle_rmsnorm.argtypes = [I, I, D, P, I, P, P, I]
        L.oracle_route.argtypes = [I, I, I, I, D, D, P, I, P, P, P, P, P, P, P, I]
        L.oracle_forward.argtypes = [I, P, I, I, I, I, I, D, D, P, I, P, P, P, P, P, I,
                                     P, P, P, P, P, P, I]
        L.oracle_expert.argtypes = [I, I, I, P, P, P, I, P, P, I, P, I]
        L.oracle_quant.argtypes = [I, I, P, P, P, P, I]
        L.oracle_e4m3.argtypes = [I, P, P, P, P]
        L.oracle_dispatch.argtypes = [I, I, I, P, P, P, P]
        L.oracle_set_threads.argtypes = [I]
        L.oracle_dense_ffn.argtypes = [I, I, I, D, P, I, P, P, P, I, P, I]
        L.oracle_shortconv.argtypes = [I, I, I, D, P, I, P, P, P, I, P, P, P, P, I]
        L.oracle_dense_ffn.restype = I
        L.oracle_shortconv.restype = I
        for f in (L.oracle_rmsnorm, L.oracle_route, L.oracle_forward, L.oracle_expert,
                  L.oracle_quant, L.oracle_e4m3, L.oracle_dispatch, L.oracle_set_threads,
                  L.oracle_num_mutations):
            f.restype = I
        _lib = L
    return _lib


def set_threads(n: int = 0) -> int:
    """Sets the OpenMP thread count (n > 0) and returns the count in use."""
    return lib().oracle_set_threads(int(n))


def _raw(t: torch.Tensor):
    """(keep-alive tensor, pointer, dtype code) for a CPU tensor's stored values."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t, t.data_ptr(), F32
    if t.dtype == torch.bfloat16:
        return t, t.data_ptr(), BF16
    if t.dtype == torch.float64:
        return t, t.data_ptr(), F64
    if t.dtype == torch.float8_e4m3fn:
        return t, t.data_ptr(), E4M3
    raise TypeError(f"unsupported dtype {t.dtype}")


def _f32(t: torch.Tensor) -> torch.Tensor:
    t = t.detach().cpu().contiguous()
    assert t.dtype == torch.float32, t.dtype
    return t


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"{what} failed with code {rc}")


def rmsnorm(x, gain, eps, mutation=0) -> np.ndarray:
    xk, xp, xdt = _raw(x)
    g = _f32(gain)
    N, d = xk.shape
    xn = np.zeros((N, d), np.float64)
    _check(lib().oracle_rmsnorm(N, d, eps, xp, xdt, g.data_ptr(), xn.ctypes.data, mutation),
           "oracle_rmsnorm")
    return xn


def route(x, layer, k, eps, routed_scale=1.0, mutation=0):
    """Returns dict(idx[N,k] int32, w[N,k] f64, s[N,E] f64, margin[N] f64)."""
    xk, xp, xdt = _raw(x)
    g, rw, b = _f32(layer["norm_gain"]), _f32(layer["router_w"]), _f32(layer["bias"])
    N, d = xk.shape
    E = rw.shape[0]
    idx = np.zeros((N, k), np.int32)
    w = np.zeros((N, k), np.float64)
    s = np.zeros((N, E), np.float64)
    margin = np.zeros(N, np.float64)
    _check(lib().oracle_route(N, d, E, k, eps, routed_scale, xp, xdt, g.data_ptr(),
                              rw.data_ptr(), b.data_ptr(), idx.ctypes.data, w.ctypes.data,
                              s.ctypes.data, margin.ctypes.data, mutation), "oracle_route")
    return {"idx": idx, "w": w, "s": s, "margin": margin}


def _scales(layer, wdt):
    """(keep-alive list, gate/up scale pointer, down scale pointer): the FP8_BLOCK
    block scales for e4m3 weights, null pointers otherwise."""
    if wdt != E4M3:
        return [], None, None
    sg, sd = _f32(layer["w_gate_up_scale"]), _f32(layer["w_down_scale"])
    return [sg, sd], sg.data_ptr(), sd.data_ptr()


def forward(x, layer, k, eps, routed_scale=1.0, tokens=None, forced=None, mutation=0):
    """Block output (x + MoE(RMSNorm(x))) in f64 for the listed tokens (all if None).

    forced: optional int array [n, k] of expert indices (slot order) to use
    instead of the oracle's own selection for those tokens.
    e4m3 expert weights (torch.float8_e4m3fn) select the FP8_BLOCK experts;
    the layer then also holds "w_gate_up_scale" [E][2I/128][d/128] and
    "w_down_scale" [E][d/128][I/128] (float32).
    Returns dict(out[n,d] f64, idx[n,k], w[n,k], tokens[n]).
    """
    xk, xp, xdt = _raw(x)
    g, rw, b = _f32(layer["norm_gain"]), _f32(layer["router_w"]), _f32(layer["bias"])
    wgu, wgp, wdt = _raw(layer["w_gate_up"])
    wd, wdp, wdt2 = _raw(layer["w_down"])
    assert wdt == wdt2
    keep, sgp, sdp = _scales(layer, wdt)
    N, d = xk.shape
    E = rw.shape[0]
    I = wgu.shape[1] // 2
    if tokens is None:
        tokens = np.arange(N, dtype=np.int64)
    tokens = np.ascontiguousarray(np.asarray(tokens, dtype=np.int64))
    n = tokens.shape[0]
    fptr = None
    if forced is not None:
        forced = np.ascontiguousarray(np.asarray(forced, dtype=np.int32))
        assert forced.shape == (n, k)
        fptr = forced.ctypes.data
    out = np.zeros((n, d), np.float64)
    idx = np.zeros((n, k), np.int32)
    w = np.zeros((n, k), np.float64)
    _check(lib().oracle_forward(n, tokens.ctypes.data, N, d, E, k, I, eps, routed_scale,
                                xp, xdt, g.data_ptr(), rw.data_ptr(), b.data_ptr(),
                                wgp, wdp, wdt, sgp, sdp, fptr, out.ctypes.data,
                                idx.ctypes.data, w.ctypes.data, mutation), "oracle_forward")
    del keep
    return {"out": out, "idx": idx, "w": w, "tokens": tokens}


def expert(xin, layer, e, mutation=0) -> np.ndarray:
    """Expert e of the layer alone on input rows xin[n][d] (f64): y[n][d] f64.
    For e4m3 weights the rows are quantised per group of 128 first."""
    xin = np.ascontiguousarray(np.asarray(xin, dtype=np.float64))
    wgu, wgp, wdt = _raw(layer["w_gate_up"])
    wd, wdp, _ = _raw(layer["w_down"])
    keep, sgp, sdp = _scales(layer, wdt)
    n, d = xin.shape
    I = wgu.shape[1] // 2
    y = np.zeros((n, d), np.float64)
    _check(lib().oracle_expert(n, d, I, xin.ctypes.data, wgp, wdp, wdt, sgp, sdp, int(e),
                               y.ctypes.data, mutation), "oracle_expert")
    del keep
    return y


def quant(v, mutation=0):
    """FP8_BLOCK activation quantisation of rows v[n][m] in groups of 128:
    dict(codes uint8 [n][m], scales f32 [n][ceil(m/128)], deq f64 [n][m])."""
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float64))
    n, m = v.shape
    ng = (m + 127) // 128
    codes = np.zeros((n, m), np.uint8)
    scales = np.zeros((n, ng), np.float32)
    deq = np.zeros((n, m), np.float64)
    _check(lib().oracle_quant(n, m, v.ctypes.data, codes.ctypes.data, scales.ctypes.data,
                              deq.ctypes.data, mutation), "oracle_quant")
    return {"codes": codes, "scales": scales, "deq": deq}


def e4m3_encode(f) -> np.ndarray:
    """e4m3 codes (uint8) of float32 values: nearest, ties to even, saturating."""
    f = np.ascontiguousarray(np.asarray(f, dtype=np.float32))
    codes = np.zeros(f.shape, np.uint8)
    _check(lib().oracle_e4m3(f.size, f.ctypes.data, codes.ctypes.data, None, None), "oracle_e4m3")
    return codes


def e4m3_value(codes) -> np.ndarray:
    """The value (f64) of each e4m3 code."""
    codes = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8))
    v = np.zeros(codes.shape, np.float64)
    _check(lib().oracle_e4m3(codes.size, None, None, codes.ctypes.data, v.ctypes.data),
           "oracle_e4m3")
    return v


def dispatch(idx: np.ndarray, n_experts: int):
    """Counting sort of assignments by expert: dict(counts, offsets, perm)."""
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
    N, k = idx.shape
    counts = np.zeros(n_experts, np.int32)
    offsets = np.zeros(n_experts + 1, np.int32)
    perm = np.zeros(N * k, np.int32)
    _check(lib().oracle_dispatch(N, n_experts, k, idx.ctypes.data, counts.ctypes.data,
                                 offsets.ctypes.data, perm.ctypes.data), "oracle_dispatch")
    return {"counts": counts, "offsets": offsets, "perm": perm}


# ---------------------------------------------------------------- neighbours
def dense_ffn(x, layer, eps, mutation=0) -> np.ndarray:
    """Dense feed-forward block: x + down(silu(gate xn) * (up xn)), xn =
    RMSNorm(x) * norm_gain; layer holds norm_gain [d] f32, w_gate_up [2I,d]
    and w_down [d,I] (f32 or bf16). Returns out [N,d] f64."""
    xk, xp, xdt = _raw(x)
    g = _f32(layer["norm_gain"])
    wgu, wgp, wdt = _raw(layer["w_gate_up"])
    wd, wdp, wdt2 = _raw(layer["w_down"])
    assert wdt == wdt2
    N, d = xk.shape
    I = wgu.shape[0] // 2
    out = np.zeros((N, d), np.float64)
    _check(lib().oracle_dense_ffn(N, d, I, eps, xp, xdt, g.data_ptr(), wgp, wdp, wdt,
                                  out.ctypes.data, mutation), "oracle_dense_ffn")
    return out


def shortconv(x, layer, eps, state_in=None, mutation=0):
    """Short-convolution block on x [B,T,d]: x + w_out (u * conv3(g * v)),
    [g; u; v] = w_in RMSNorm(x) * norm_gain. layer holds norm_gain [d] f32,
    w_in [3d,d] and w_out [d,d] (f32 or bf16), conv [d,3] f32 indexed by lag.
    state_in: optional [B,2,d] a vectors of positions -2, -1 per sequence.
    Returns (out [B,T,d] f64, state_out [B,2,d] f64)."""
    xk, xp, xdt = _raw(x)
    B, T, d = xk.shape
    g = _f32(layer["norm_gain"])
    win, wip, wdt = _raw(layer["w_in"])
    wo, wop, wdt2 = _raw(layer["w_out"])
    assert wdt == wdt2
    kc = _f32(layer["conv"])
    assert tuple(kc.shape) == (d, 3)
    sp = None
    if state_in is not None:
        st = np.ascontiguousarray(np.asarray(state_in, dtype=np.float64))
        assert st.shape == (B, 2, d)
        sp = st.ctypes.data
    out = np.zeros((B, T, d), np.float64)
    so = np.zeros((B, 2, d), np.float64)
    _check(lib().oracle_shortconv(B, T, d, eps, xp, xdt, g.data_ptr(), wip, wop, wdt,
                                  kc.data_ptr(), sp, out.ctypes.data, so.ctypes.data, mutation),
           "oracle_shortconv")
    return out, so
