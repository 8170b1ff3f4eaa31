"""moe_route_noalloc, the routing entry point that allocates nothing, against
the routing of a context's forward (moe_forward + moe_debug_routing) and
against the fp64 oracle.

Its users are callers that cannot allocate device memory where they route:
work recorded into a CUDA graph, serving loops that forbid allocator calls
(they can synchronise the device), or hosts whose memory planner owns all
device memory. Its scratch is a fixed array inside the library, so two calls
in a row must each give the full, correct result (nothing may depend on what
the previous call left in the array). Where the two routers differ in kernel
(4096 tokens: the tiled SIMT router here, the tensor-core router in a bf16
context), indices are compared exactly only on tokens whose oracle margin
exceeds 1e-3, as everywhere else; the others are checked by the oracle's
near-tie rule. Kept in its own file so that it runs after every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import sigmoid_bias_top_b200 as sb
from sigmoid_bias_top_b200 import MoeLayer, workloads as W
from tests import parity as PA

pytestmark = pytest.mark.gpu

CASES = {
    "decode_32": W.DECODE.scaled(n_tokens=32),
    "decode_4096": W.DECODE.scaled(n_tokens=4096),
    "ragged_100": W.DECODE.scaled(n_tokens=100),
    "ragged_4095": W.DECODE.scaled(n_tokens=4095),
    "experts_16": W.DECODE.scaled(n_tokens=77, n_experts=16, d=512, d_ff=256),
    "tiny_f32": W.TINY_F32,
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_noalloc_routing_matches_context_forward_twice(case):
    w = CASES[case]
    n = w.n_tokens
    layer = W.make_layer(w, 0, "cuda")
    x = W.make_x(w, "cuda")
    m = MoeLayer(layer, w.top_k, w.eps, w.routed_scale, max_tokens=n)
    m(x)
    ref = m.debug_routing(n)
    torch.cuda.synchronize()
    assert m.status() == 0
    x_cpu, l_cpu = x.cpu(), PA.to_cpu_layer(layer)
    oref = PA.check_routing(x_cpu, l_cpu, w.top_k, w.eps, w.routed_scale, ref)[0]
    clear = torch.from_numpy(oref["margin"] > PA.MARGIN).cuda()
    L = sb.lib()
    stream = torch.cuda.current_stream().cuda_stream
    dt = sb.MOE_F32 if x.dtype == torch.float32 else sb.MOE_BF16
    for call in range(2):
        idx = torch.full((n, w.top_k), -1, dtype=torch.int32, device="cuda")
        wt = torch.full((n, w.top_k), float("nan"), dtype=torch.float32, device="cuda")
        rc = L.moe_route_noalloc(x.data_ptr(), dt, layer["norm_gain"].data_ptr(),
                                 layer["router_w"].data_ptr(), layer["bias"].data_ptr(),
                                 n, w.d, w.n_experts, w.top_k, w.eps, w.routed_scale,
                                 idx.data_ptr(), wt.data_ptr(), ctypes.c_void_p(stream))
        assert rc == 0, sb.strerror(rc)
        torch.cuda.synchronize()
        assert torch.equal(idx[clear], ref["idx"][clear]), f"call {call}: expert indices differ"
        same = (idx == ref["idx"]).all(1)
        torch.testing.assert_close(wt[same], ref["w"][same], rtol=1e-6, atol=1e-7)
        PA.check_routing(x_cpu, l_cpu, w.top_k, w.eps, w.routed_scale, {"idx": idx, "w": wt})
    m.close()


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
