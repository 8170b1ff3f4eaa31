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

F32, BF16, F64 = 0, 1, 2

MUTATIONS = {
    "none": 0, "biased_weights": 1, "softmax": 2, "bias_before_act": 3,
    "no_eps": 4, "no_gain": 5, "silu_on_up": 6, "tie_high": 7,
    "no_residual": 8, "mean_not_sum": 9, "slot_swap": 10, "down_transposed": 11,
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
                                     P, P, P, P, I]
        L.oracle_dispatch.argtypes = [I, I, I, P, P, P, P]
        L.oracle_set_threads.argtypes = [I]
        for f in (L.oracle_rmsnorm, L.oracle_route, L.oracle_forward,
                  L.oracle_dispatch, L.oracle_set_threads, L.oracle_num_mutations):
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


def forward(x, layer, k, eps, routed_scale=1.0, tokens=None, forced=None, mutation=0):
    """Block output (x + MoE(RMSNorm(x))) in f64 for the listed tokens (all if None).

    forced: optional int array [n, k] of expert indices (slot order) to use
    instead of the oracle's own selection for those tokens.
    Returns dict(out[n,d] f64, idx[n,k], w[n,k], tokens[n]).
    """
    xk, xp, xdt = _raw(x)
    g, rw, b = _f32(layer["norm_gain"]), _f32(layer["router_w"]), _f32(layer["bias"])
    wgu, wgp, wdt = _raw(layer["w_gate_up"])
    wd, wdp, wdt2 = _raw(layer["w_down"])
    assert wdt == wdt2
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
                                wgp, wdp, wdt, fptr, out.ctypes.data, idx.ctypes.data,
                                w.ctypes.data, mutation), "oracle_forward")
    return {"out": out, "idx": idx, "w": w, "tokens": tokens}


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
