"""ctypes binding of the dense feed-forward block and the short-convolution
block (include/block.h): argument marshalling only; every step runs in
libmoe.so's CUDA kernels.

"LFM2.5-24B-A2B: Biased Routing, Short Convolutions and Ten KV Caches"
(flozi.net, English page), sections "The exact checkpoint" (the first two
layers are dense and convolutional) and "A short convolution is a local
mixer, not an embedding lookup".
"""
from __future__ import annotations

import ctypes
from typing import Dict, Optional

from . import MOE_BF16, _check, _stream_ptr, lib as _moe_lib


class DenseWeights(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("norm_gain", ctypes.c_void_p),
                ("w_gate_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p)]


class ConvWeights(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("norm_gain", ctypes.c_void_p),
                ("w_in", ctypes.c_void_p), ("conv", ctypes.c_void_p),
                ("w_out", ctypes.c_void_p)]


_bound = False


def lib():
    global _bound
    L = _moe_lib()
    if not _bound:
        P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.moe_dense_create.argtypes = [I, I, F, ctypes.POINTER(DenseWeights), I,
                                       ctypes.POINTER(P)]
        L.moe_conv_create.argtypes = [I, F, ctypes.POINTER(ConvWeights), I, ctypes.POINTER(P)]
        L.moe_dense_forward.argtypes = [P, P, P, I, P]
        L.moe_conv_forward.argtypes = [P, P, P, I, I, P, P, P]
        L.moe_block_status.argtypes = [P]
        L.moe_block_destroy.argtypes = [P]
        L.moe_block_profile.argtypes = [P, I]
        L.moe_block_kernel_times.argtypes = [P, ctypes.POINTER(F), I]
        L.moe_block_kernel_name.argtypes = [P, I]
        L.moe_block_kernel_name.restype = ctypes.c_char_p
        for f in (L.moe_dense_create, L.moe_conv_create, L.moe_dense_forward,
                  L.moe_conv_forward, L.moe_block_status, L.moe_block_destroy,
                  L.moe_block_profile, L.moe_block_kernel_times):
            f.restype = I
        _bound = True
    return L


class _Block:
    _h = None

    def status(self) -> int:
        return lib().moe_block_status(self._h)

    def profile(self, enable: bool = True):
        _check(lib().moe_block_profile(self._h, int(enable)), "moe_block_profile")

    def kernel_times(self) -> Dict[str, float]:
        ms = (ctypes.c_float * 8)()
        n = lib().moe_block_kernel_times(self._h, ms, 8)
        if n < 0:
            _check(n, "moe_block_kernel_times")
        return {lib().moe_block_kernel_name(self._h, i).decode(): ms[i] for i in range(n)}

    def close(self):
        if getattr(self, "_h", None):
            rc = lib().moe_block_destroy(self._h)
            self._h = None
            _check(rc, "moe_block_destroy")

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class DenseBlock(_Block):
    """out = x + W_down(silu(W_gate xn) * (W_up xn)), xn = RMSNorm(x) * gain.
    layer: norm_gain [d] f32, w_gate_up [2I, d] and w_down [d, I] bf16."""

    def __init__(self, layer: Dict, eps: float = 1e-6, max_tokens: int = 1024):
        import torch
        wgu = layer["w_gate_up"]
        twoI, d = wgu.shape
        if wgu.dtype != torch.bfloat16:
            raise TypeError("the dense block takes bf16 matrices")
        self._keep = {n: layer[n].contiguous() for n in ("norm_gain", "w_gate_up", "w_down")}
        k = self._keep
        self._w = DenseWeights(MOE_BF16, k["norm_gain"].data_ptr(), k["w_gate_up"].data_ptr(),
                               k["w_down"].data_ptr())
        self.d, self.I, self.device = d, twoI // 2, wgu.device
        h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            _check(lib().moe_dense_create(d, self.I, eps, ctypes.byref(self._w), max_tokens,
                                          ctypes.byref(h)), "moe_dense_create")
        self._h = h

    def forward(self, x, out=None, stream=None):
        import torch
        if out is None:
            out = torch.empty_like(x)
        _check(lib().moe_dense_forward(self._h, x.data_ptr(), out.data_ptr(), x.shape[0],
                                       _stream_ptr(stream)), "moe_dense_forward")
        return out

    __call__ = forward


class ConvBlock(_Block):
    """Short-convolution block on x [B, T, d]: x + W_out(u * conv3(g * v)),
    [g; u; v] = W_in RMSNorm(x) * gain. layer: norm_gain [d] f32, w_in
    [3d, d] and w_out [d, d] bf16, conv [d, 3] f32 (by lag)."""

    def __init__(self, layer: Dict, eps: float = 1e-6, max_tokens: int = 1024):
        import torch
        w_in = layer["w_in"]
        d = w_in.shape[1]
        if w_in.dtype != torch.bfloat16:
            raise TypeError("the conv block takes bf16 matrices")
        self._keep = {n: layer[n].contiguous() for n in ("norm_gain", "w_in", "conv", "w_out")}
        k = self._keep
        self._w = ConvWeights(MOE_BF16, k["norm_gain"].data_ptr(), k["w_in"].data_ptr(),
                              k["conv"].data_ptr(), k["w_out"].data_ptr())
        self.d, self.device = d, w_in.device
        h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            _check(lib().moe_conv_create(d, eps, ctypes.byref(self._w), max_tokens,
                                         ctypes.byref(h)), "moe_conv_create")
        self._h = h

    def forward(self, x, out=None, state_in=None, state_out=None, stream=None):
        """x [B, T, d] bf16; state_in / state_out: [B, 2, d] f32 or None."""
        import torch
        B, T, d = x.shape
        if out is None:
            out = torch.empty_like(x)
        _check(lib().moe_conv_forward(self._h, x.data_ptr(), out.data_ptr(), B, T,
                                      None if state_in is None else state_in.data_ptr(),
                                      None if state_out is None else state_out.data_ptr(),
                                      _stream_ptr(stream)), "moe_conv_forward")
        return out

    __call__ = forward
