"""moe_route_noalloc, the routing entry point that allocates nothing, against
the routing of a context's forward (moe_forward + moe_debug_routing).

Its users are callers that cannot allocate device memory where they route:
work recorded into a CUDA graph, serving loops that forbid allocator calls
(they can synchronise the device), or hosts whose memory planner owns all
device memory. Its scratch is a fixed array inside the library, so two calls
in a row must each give the full, correct result (nothing may depend on what
the previous call left in the array). Kept in its own file so that it runs
after every other test.
"""
import ctypes

import pytest
import torch

import sigmoid_bias_top_b200 as sb
from sigmoid_bias_top_b200 import MoeLayer, workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n_tokens", [32, 4096])
def test_noalloc_routing_matches_context_forward_twice(n_tokens):
    w = W.DECODE.scaled(n_tokens=n_tokens)
    layer = W.make_layer(w, 0, "cuda")
    x = W.make_x(w, "cuda")
    m = MoeLayer(layer, w.top_k, w.eps, w.routed_scale, max_tokens=n_tokens)
    m(x)
    ref = m.debug_routing(n_tokens)
    torch.cuda.synchronize()
    assert m.status() == 0
    L = sb.lib()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        idx = torch.full((n_tokens, w.top_k), -1, dtype=torch.int32, device="cuda")
        wt = torch.full((n_tokens, w.top_k), float("nan"), dtype=torch.float32, device="cuda")
        rc = L.moe_route_noalloc(x.data_ptr(), sb.MOE_BF16, layer["norm_gain"].data_ptr(),
                                 layer["router_w"].data_ptr(), layer["bias"].data_ptr(),
                                 n_tokens, w.d, w.n_experts, w.top_k, w.eps, w.routed_scale,
                                 idx.data_ptr(), wt.data_ptr(), ctypes.c_void_p(stream))
        assert rc == 0, sb.strerror(rc)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref["idx"]), f"call {call}: expert indices differ"
        torch.testing.assert_close(wt, ref["w"], rtol=1e-6, atol=1e-7)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    w = W.DECODE.scaled(n_tokens=8)
    layer = W.make_layer(w, 0, "cuda")
    x = W.make_x(w, "cuda")
    L = sb.lib()
    idx = torch.empty(8, 4, dtype=torch.int32, device="cuda")
    wt = torch.empty(8, 4, dtype=torch.float32, device="cuda")
    args = (sb.MOE_BF16, layer["norm_gain"].data_ptr(), layer["router_w"].data_ptr(),
            layer["bias"].data_ptr())
    assert L.moe_route_noalloc(x.data_ptr(), *args, 4097, 2048, 64, 4, 1e-6, 1.0,
                               idx.data_ptr(), wt.data_ptr(), None) == -4
    assert L.moe_route_noalloc(x.data_ptr(), *args, 8, 4096, 64, 4, 1e-6, 1.0,
                               idx.data_ptr(), wt.data_ptr(), None) == -2
    assert L.moe_route_noalloc(x.data_ptr(), *args, 8, 2048, 128, 4, 1e-6, 1.0,
                               idx.data_ptr(), wt.data_ptr(), None) == -2
