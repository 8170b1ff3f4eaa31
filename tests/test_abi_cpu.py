"""The C-ABI library builds for sm_100a, loads without a GPU, and exports every
entry point include/moe.h declares. Host-side validation is checked where it
runs before any device call."""
import ctypes
import os
import re

import pytest
import torch

import sigmoid_bias_top_b200 as sb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names.update(re.findall(r"\b(moe_[a-z_]+)\s*\(", src))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    for n in ("moe_create", "moe_forward", "moe_destroy", "moe_ep_create", "moe_ep_dispatch",
              "moe_dense_create", "moe_conv_forward", "moe_block_destroy"):
        assert n in names, n
    L = sb.lib()
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing


def test_library_is_sm100a_build():
    data = open(sb.LIB_PATH, "rb").read()
    assert b"sm_100a" in data or b"compute_100a" in data


def test_strerror_covers_codes():
    for code, name in sb.ERRORS.items():
        msg = sb.strerror(code)
        assert msg and msg != "unknown error", (code, name)
    assert sb.strerror(12345) == "unknown error"


def _weights(dtype=sb.MOE_BF16, ptr=256):
    return sb.MoeWeights(dtype, ptr, ptr, ptr, ptr, ptr, 1.0)


def _create(d, E, I, k, w, max_tokens=16):
    h = ctypes.c_void_p(1234)
    rc = sb.lib().moe_create(d, E, I, k, 1e-6, ctypes.byref(w) if w is not None else None,
                             max_tokens, ctypes.byref(h))
    return rc, h


def test_create_validates_before_touching_the_device():
    w = _weights()
    assert _create(2048, 64, 1536, 4, None)[0] == -1            # no weights
    rc, h = _create(2048, 64, 1536, 9, w)
    assert rc == -2 and not h.value                              # k > 8, handle cleared
    assert _create(2048, 4, 1536, 5, w)[0] == -2                 # k > E
    assert _create(2048, 300, 1536, 4, w)[0] == -2               # E > 256
    assert _create(2000, 64, 1536, 4, w)[0] == -2                # bf16 d % 64
    assert _create(2048, 64, 1500, 4, w)[0] == -2                # bf16 I % 64
    assert _create(2048, 64, 1536, 4, w, max_tokens=0)[0] == -2
    assert _create(2048, 64, 1536, 4, _weights(dtype=7))[0] == -1
    assert _create(2048, 64, 1536, 4, _weights(ptr=258))[0] == -3  # misaligned
    assert _create(2048, 64, 1536, 4, _weights(ptr=0))[0] == -1    # null
    # FP8_BLOCK: whole 128 x 128 scale blocks, both scale arrays given and aligned
    f8 = _weights(dtype=sb.MOE_FP8_BLOCK)
    assert _create(2048, 64, 1536, 4, f8)[0] == -1               # no block scales
    f8.w_gate_up_scale, f8.w_down_scale = 256, 256
    assert _create(2112, 64, 1536, 4, f8)[0] == -2               # d % 128
    assert _create(2048, 64, 1600, 4, f8)[0] == -2               # I % 128
    f8.w_down_scale = 260
    assert _create(2048, 64, 1536, 4, f8)[0] == -3               # misaligned scales


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU answer")
def test_create_without_gpu_reports_no_device():
    rc, h = _create(256, 16, 192, 4, _weights(dtype=sb.MOE_F32))
    assert rc == -9 and not h.value


def test_route_noalloc_takes_the_storage_type_of_x():
    """The no-allocation router takes x's own dtype (f32 or bf16); the
    FP8_BLOCK layer dtype, which describes expert weights, is refused before
    any device work."""
    L = sb.lib()
    args = (256, 1, 256, 256, 256, 8, 256, 16, 4, 1e-6, 1.0, 256, 256, None)
    assert L.moe_route_noalloc(args[0], sb.MOE_FP8_BLOCK, *args[2:]) == -1


def test_route_noalloc_refuses_shapes_before_device_work():
    """Shapes outside what moe_create takes are refused on the host: bf16 rows
    need d % 64 == 0 (the router copies whole row groups in 16-byte units),
    fp32 rows d % 4 == 0; sizes beyond the fixed scratch are refused too."""
    L = sb.lib()

    def call(dtype, n, d, E, k):
        return L.moe_route_noalloc(256, dtype, 256, 256, 256, n, d, E, k, 1e-6, 1.0, 256, 256,
                                   None)
    assert call(sb.MOE_BF16, 7, 100, 16, 4) == -2       # d % 8 == 4: odd row groups
    assert call(sb.MOE_BF16, 7, 96, 16, 4) == -2        # d % 64 != 0
    assert call(sb.MOE_F32, 7, 102, 16, 4) == -2        # d % 4 != 0
    assert call(sb.MOE_F32, 7, 256, 16, 9) == -2        # k > 8
    assert call(sb.MOE_F32, 7, 256, 4, 5) == -2         # k > E
    assert call(sb.MOE_BF16, 4097, 2048, 64, 4) == -4   # beyond the scratch's tokens
    assert call(sb.MOE_BF16, 8, 4096, 64, 4) == -2      # beyond its width
    assert call(sb.MOE_BF16, 8, 2048, 128, 4) == -2     # beyond its experts
    assert call(sb.MOE_BF16, 0, 2048, 64, 4) == 0       # empty batch: nothing to do


def test_route_noalloc_binding_checks_tensors():
    """The Python binding refuses other dtypes and non-contiguous tensors
    before calling the library."""
    layer = {"norm_gain": torch.ones(64), "router_w": torch.zeros(8, 64), "bias": torch.zeros(8)}
    with pytest.raises(TypeError):
        sb.route_noalloc(torch.zeros(4, 64, dtype=torch.float16), layer, 2)
    with pytest.raises(ValueError):
        sb.route_noalloc(torch.zeros(64, 4).t(), layer, 2)


def test_calls_on_null_handle_are_rejected():
    L = sb.lib()
    assert L.moe_forward(None, None, None, 1, None) == -1
    assert L.moe_status(None) == -1
    assert L.moe_destroy(None) == 0
    assert L.moe_profile(None, 1) == -1


def test_ep_create_validates_before_touching_the_device():
    L = sb.lib()
    h = ctypes.c_void_p(99)
    w = _weights()

    def create(d=2048, E=64, I=1536, k=4, first=0, n_local=8, cap=1024, ww=w):
        return L.moe_ep_create(d, E, I, k, 1e-6, ctypes.byref(ww), 16, first, n_local, cap,
                               ctypes.byref(h))
    assert create(first=60, n_local=8) == -2 and not h.value    # block past E
    assert create(n_local=0) == -2
    assert create(cap=0) == -2
    assert create(ww=_weights(dtype=sb.MOE_FP8_BLOCK)) == -1    # bf16 / f32 only
    assert create(d=2000) == -2


def test_block_create_validates_before_touching_the_device():
    from sigmoid_bias_top_b200 import blocks as B
    L = B.lib()
    h = ctypes.c_void_p(99)
    dw = B.DenseWeights(sb.MOE_BF16, 256, 256, 256)
    assert L.moe_dense_create(2000, 6144, 1e-6, ctypes.byref(dw), 16, ctypes.byref(h)) == -2
    assert L.moe_dense_create(2048, 6100, 1e-6, ctypes.byref(dw), 16, ctypes.byref(h)) == -2
    assert L.moe_dense_create(2048, 6144, 1e-6, ctypes.byref(B.DenseWeights(sb.MOE_F32, 256,
                              256, 256)), 16, ctypes.byref(h)) == -1
    assert L.moe_dense_create(2048, 6144, 1e-6, ctypes.byref(B.DenseWeights(sb.MOE_BF16, 258,
                              256, 256)), 16, ctypes.byref(h)) == -3
    cw = B.ConvWeights(sb.MOE_BF16, 256, 256, 256, 256)
    assert L.moe_conv_create(100, 1e-6, ctypes.byref(cw), 16, ctypes.byref(h)) == -2
    assert L.moe_conv_create(2048, 1e-6, ctypes.byref(B.ConvWeights(sb.MOE_BF16, 256, 256, 0,
                             256)), 16, ctypes.byref(h)) == -1
    assert not h.value
    assert L.moe_block_destroy(None) == 0 and L.moe_block_status(None) == -1
