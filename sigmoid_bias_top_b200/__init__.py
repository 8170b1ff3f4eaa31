"""B200 (sm_100a) sigmoid-bias top-k mixture-of-experts feed-forward block.

Thin ctypes binding of libmoe.so, the C ABI declared in include/moe.h. It only
marshals torch tensors (device memory, streams) into the C calls: every step
of the layer runs in the library's CUDA kernels. There is no CPU path; if the
library is missing or no sm_100 GPU is present, the calls raise.

Layer (see include/moe.h): out = x + sum_j w_j * Expert_{S_j}(RMSNorm(x)), with
the top-k set S chosen on sigmoid(router logits) + expert bias and the weights
w taken from the unbiased sigmoid scores normalised by (their sum + eps).
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_F32, MOE_BF16, MOE_FP8_BLOCK = 0, 1, 2
ERRORS = {
    0: "MOE_OK", -1: "MOE_ERR_INVALID_ARG", -2: "MOE_ERR_UNSUPPORTED_SHAPE",
    -3: "MOE_ERR_ALIGNMENT", -4: "MOE_ERR_TOO_MANY_TOKENS", -5: "MOE_ERR_OOM",
    -6: "MOE_ERR_CUDA", -7: "MOE_ERR_DEVICE_TIMEOUT", -8: "MOE_ERR_DEVICE_BOUNDS",
    -9: "MOE_ERR_NO_DEVICE",
}


class MoeError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {ERRORS.get(code, code)} ({strerror(code)})")


class MoeWeights(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("norm_gain", ctypes.c_void_p),
                ("router_w", ctypes.c_void_p), ("expert_bias", ctypes.c_void_p),
                ("w_gate_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p),
                ("routed_scale", ctypes.c_float), ("w_gate_up_scale", ctypes.c_void_p),
                ("w_down_scale", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C-ABI library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m sigmoid_bias_top_b200._build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.moe_create.argtypes = [I, I, I, I, F, ctypes.POINTER(MoeWeights), I,
                                 ctypes.POINTER(P)]
        L.moe_forward.argtypes = [P, P, P, I, P]
        L.moe_forward_host.argtypes = [P, P, P, I, P]
        L.moe_destroy.argtypes = [P]
        L.moe_status.argtypes = [P]
        L.moe_debug_routing.argtypes = [P, P, P, P, P, P]
        L.moe_debug_fp8_rows.argtypes = [P, P, P, P]
        L.moe_profile.argtypes = [P, I]
        L.moe_kernel_times.argtypes = [P, ctypes.POINTER(F), I]
        L.moe_kernel_name.argtypes = [P, I]
        L.moe_kernel_name.restype = ctypes.c_char_p
        L.moe_launches_per_forward.argtypes = [P, I]
        L.moe_selftest_timeout.argtypes = [P, I, P]
        L.moe_selftest_fp8_divide.argtypes = [P, P, P, P, I, P]
        L.moe_selftest_fp8_divide.restype = I
        L.moe_route_noalloc.argtypes = [P, I, P, P, P, I, I, I, I, F, F, P, P, P]
        L.moe_route_noalloc.restype = I
        L.moe_strerror.argtypes = [I]
        L.moe_strerror.restype = ctypes.c_char_p
        # expert parallelism (ep.py)
        L.moe_ep_create.argtypes = [I, I, I, I, F, ctypes.POINTER(MoeWeights), I, I, I, I,
                                    ctypes.POINTER(P)]
        L.moe_ep_dispatch.argtypes = [P, P, I, P, P]
        L.moe_ep_buffers.argtypes = [P, ctypes.POINTER(P), ctypes.POINTER(P),
                                     ctypes.POINTER(P), ctypes.POINTER(P)]
        L.moe_ep_experts.argtypes = [P, P, P]
        L.moe_ep_combine.argtypes = [P, P, P, P]
        L.moe_ep_debug_routing.argtypes = [P, P, P, P, P, P]
        L.moe_ep_status.argtypes = [P]
        L.moe_ep_destroy.argtypes = [P]
        for f in (L.moe_ep_create, L.moe_ep_dispatch, L.moe_ep_buffers, L.moe_ep_experts,
                  L.moe_ep_combine, L.moe_ep_debug_routing, L.moe_ep_status,
                  L.moe_ep_destroy):
            f.restype = I
        for f in (L.moe_create, L.moe_forward, L.moe_forward_host, L.moe_destroy,
                  L.moe_status, L.moe_debug_routing, L.moe_debug_fp8_rows, L.moe_profile,
                  L.moe_kernel_times,
                  L.moe_launches_per_forward, L.moe_selftest_timeout):
            f.restype = I
        _lib = L
    return _lib


def strerror(code: int) -> str:
    return lib().moe_strerror(int(code)).decode()


def _check(rc: int, what: str):
    if rc != 0:
        raise MoeError(rc, what)


def _stream_ptr(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def route_noalloc(x, layer: Dict, top_k: int, eps: float = 1e-6, routed_scale: float = 1.0,
                  idx=None, w=None, stream=None):
    """Routing without device allocation (moe_route_noalloc): returns (idx, w).

    For callers that must not allocate device memory at this point (stream
    capture, allocator-free serving loops); idx and w may be passed in
    preallocated so that the call itself allocates nothing."""
    import torch
    if x.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(f"x must be float32 or bfloat16, got {x.dtype}")
    if x.dim() != 2 or not x.is_contiguous() or not x.is_cuda:
        raise ValueError("x must be a contiguous [n, d] CUDA tensor")
    n, d = x.shape
    E = layer["router_w"].shape[0]
    for name, want in (("norm_gain", (d,)), ("router_w", (E, d)), ("bias", (E,))):
        t = layer[name]
        if (t.dtype != torch.float32 or tuple(t.shape) != want or not t.is_contiguous()
                or t.device != x.device):
            raise ValueError(f"{name} must be a contiguous float32 {want} tensor on {x.device}")
    if idx is None:
        idx = torch.empty(n, top_k, dtype=torch.int32, device=x.device)
    if w is None:
        w = torch.empty(n, top_k, dtype=torch.float32, device=x.device)
    for name, t, dt_ in (("idx", idx, torch.int32), ("w", w, torch.float32)):
        if (t.dtype != dt_ or tuple(t.shape) != (n, top_k) or not t.is_contiguous()
                or t.device != x.device):
            raise ValueError(f"{name} must be a contiguous {dt_} ({n}, {top_k}) tensor on {x.device}")
    dt = MOE_BF16 if x.dtype == torch.bfloat16 else MOE_F32
    _check(lib().moe_route_noalloc(x.data_ptr(), dt, layer["norm_gain"].data_ptr(),
                                   layer["router_w"].data_ptr(), layer["bias"].data_ptr(), n, d, E,
                                   top_k, eps, routed_scale, idx.data_ptr(), w.data_ptr(),
                                   _stream_ptr(stream)), "moe_route_noalloc")
    return idx, w


def selftest_fp8_divide(a, b, stream=None):
    """(q, q_ref) for fp32 device tensors a, b of one shape: q = a / b as the
    FP8 quantisers form it, q_ref = the IEEE quotient (moe_selftest_fp8_divide)."""
    import torch
    if a.dtype != torch.float32 or b.dtype != torch.float32 or a.shape != b.shape:
        raise ValueError("a and b: fp32 tensors of one shape")
    a, b = a.contiguous(), b.contiguous()
    q, q_ref = torch.empty_like(a), torch.empty_like(a)
    _check(lib().moe_selftest_fp8_divide(a.data_ptr(), b.data_ptr(), q.data_ptr(),
                                         q_ref.data_ptr(), a.numel(), _stream_ptr(stream)),
           "moe_selftest_fp8_divide")
    return q, q_ref


class MoeLayer:
    """One MoE block bound to device weights (borrowed, kept alive here).

    layer: dict with norm_gain [d] f32, router_w [E,d] f32, bias [E] f32,
    w_gate_up [E,2I,d] and w_down [E,d,I] (both f32 or bf16), on one CUDA device.
    FP8_BLOCK layers hold e4m3 (torch.float8_e4m3fn) expert matrices plus
    w_gate_up_scale [E,2I/128,d/128] and w_down_scale [E,d/128,I/128] (f32);
    their x and out are bf16.
    """

    def __init__(self, layer: Dict, top_k: int, eps: float = 1e-6,
                 routed_scale: float = 1.0, max_tokens: int = 1024):
        import torch
        wgu, wd = layer["w_gate_up"], layer["w_down"]
        E, twoI, d = wgu.shape
        I = twoI // 2
        names = ["norm_gain", "router_w", "bias", "w_gate_up", "w_down"]
        if wgu.dtype == torch.bfloat16:
            dt = MOE_BF16
        elif wgu.dtype == torch.float32:
            dt = MOE_F32
        elif wgu.dtype == torch.float8_e4m3fn:
            dt = MOE_FP8_BLOCK
            names += ["w_gate_up_scale", "w_down_scale"]
        else:
            raise TypeError(f"expert weights must be f32, bf16 or e4m3, got {wgu.dtype}")
        self._keep = {n: layer[n].contiguous() for n in names}
        for n, t in self._keep.items():
            if not t.is_cuda:
                raise ValueError(f"{n} must be a CUDA tensor")
        self.d, self.E, self.I, self.k = d, E, I, top_k
        self.dtype = wgu.dtype
        self.fp8 = dt == MOE_FP8_BLOCK
        self.max_tokens = max_tokens
        k = self._keep
        self._w = MoeWeights(dt, k["norm_gain"].data_ptr(), k["router_w"].data_ptr(),
                             k["bias"].data_ptr(), k["w_gate_up"].data_ptr(),
                             k["w_down"].data_ptr(), routed_scale,
                             k["w_gate_up_scale"].data_ptr() if self.fp8 else None,
                             k["w_down_scale"].data_ptr() if self.fp8 else None)
        h = ctypes.c_void_p()
        with torch.cuda.device(wgu.device):
            _check(lib().moe_create(d, E, I, top_k, eps, ctypes.byref(self._w), max_tokens,
                                    ctypes.byref(h)), "moe_create")
        self._h = h
        self.device = wgu.device

    def forward(self, x, out=None, stream=None):
        import torch
        n = x.shape[0]
        if out is None:
            out = torch.empty_like(x)
        _check(lib().moe_forward(self._h, x.data_ptr(), out.data_ptr(), n,
                                 _stream_ptr(stream)), "moe_forward")
        return out

    __call__ = forward

    def forward_host(self, x_host, out_host, stream=None):
        """x_host, out_host: CPU tensors (pinned for asynchronous copies)."""
        _check(lib().moe_forward_host(self._h, x_host.data_ptr(), out_host.data_ptr(),
                                      x_host.shape[0], _stream_ptr(stream)), "moe_forward_host")
        return out_host

    def debug_routing(self, n_tokens: int, stream=None):
        """Routing of the last forward: dict(idx, w, perm, offsets) device tensors."""
        import torch
        dev = self.device
        idx = torch.empty(n_tokens, self.k, dtype=torch.int32, device=dev)
        w = torch.empty(n_tokens, self.k, dtype=torch.float32, device=dev)
        perm = torch.empty(n_tokens * self.k, dtype=torch.int32, device=dev)
        offsets = torch.empty(self.E + 1, dtype=torch.int32, device=dev)
        _check(lib().moe_debug_routing(self._h, idx.data_ptr(), w.data_ptr(), perm.data_ptr(),
                                       offsets.data_ptr(), _stream_ptr(stream)),
               "moe_debug_routing")
        return {"idx": idx, "w": w, "perm": perm, "offsets": offsets}

    def debug_fp8_rows(self, n_tokens: int, stream=None):
        """FP8_BLOCK layers: the last forward's grouped e4m3 input rows (uint8
        codes [n*k, d], in the order of debug_routing's perm) and their group
        scales [n*k, d/128] f32, as device tensors."""
        import torch
        rows = n_tokens * self.k
        codes = torch.empty(rows, self.d, dtype=torch.uint8, device=self.device)
        scales = torch.empty(rows, self.d // 128, dtype=torch.float32, device=self.device)
        _check(lib().moe_debug_fp8_rows(self._h, codes.data_ptr(), scales.data_ptr(),
                                        _stream_ptr(stream)), "moe_debug_fp8_rows")
        return {"codes": codes, "scales": scales}

    def status(self) -> int:
        return lib().moe_status(self._h)

    def profile(self, enable: bool = True):
        _check(lib().moe_profile(self._h, int(enable)), "moe_profile")

    def kernel_times(self) -> Dict[str, float]:
        ms = (ctypes.c_float * 16)()
        n = lib().moe_kernel_times(self._h, ms, 16)
        if n < 0:
            raise MoeError(n, "moe_kernel_times")
        return {lib().moe_kernel_name(self._h, i).decode(): ms[i] for i in range(n)}

    def launches_per_forward(self, n_tokens: int) -> int:
        return lib().moe_launches_per_forward(self._h, n_tokens)

    def selftest_timeout(self, timeout_us: int, stream=None):
        _check(lib().moe_selftest_timeout(self._h, timeout_us, _stream_ptr(stream)),
               "moe_selftest_timeout")

    def close(self):
        if getattr(self, "_h", None):
            rc = lib().moe_destroy(self._h)
            self._h = None
            _check(rc, "moe_destroy")

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
