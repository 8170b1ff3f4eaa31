"""Expert parallelism through the C ABI (moe_ep_*) on one GPU: W ranks, each
an EpShard holding E/W experts, run one forward in turn with the exchanges
done as local copies (ep.emulate_ep_forward, the same plans the NCCL path
uses). Every rank's routing, dispatch and outputs are checked against the
fp64 oracle, and against the single-context forward of the same tokens."""
import numpy as np
import pytest
import torch

from sigmoid_bias_top_b200 import MoeLayer, ep, workloads as W
from tests import parity as PA

pytestmark = pytest.mark.gpu


def _shards(w, layer, world, max_tokens):
    El = w.n_experts // world
    shards = []
    for r in range(world):
        loc = dict(layer, w_gate_up=layer["w_gate_up"][r * El:(r + 1) * El],
                   w_down=layer["w_down"][r * El:(r + 1) * El])
        shards.append(ep.EpShard(loc, w.n_experts, r * El, w.top_k, w.eps, w.routed_scale,
                                 max_tokens=max_tokens, world=world))
    return shards


@pytest.mark.parametrize("case,world", [("decode", 8), ("mid", 8), ("tiny_f32", 4)])
def test_emulated_ranks_match_the_oracle(case, world):
    w = {"decode": W.DECODE, "mid": W.DECODE.scaled(n_tokens=1024),
         "tiny_f32": W.TINY_F32}[case]
    layer = W.make_layer(w, 0, "cuda")
    N = w.n_tokens
    xs = [W.make_x(w, "cuda", seed=w.seed + 31 * r) for r in range(world)]
    outs = [torch.empty_like(x) for x in xs]
    shards = _shards(w, layer, world, N)
    ep.emulate_ep_forward(shards, xs, outs)
    torch.cuda.synchronize()
    l_cpu = PA.to_cpu_layer(layer)
    single = MoeLayer(layer, w.top_k, w.eps, w.routed_scale, max_tokens=N)
    for r, (s, x, o) in enumerate(zip(shards, xs, outs)):
        assert s.status() == 0
        rt = s.debug_routing(N)
        torch.cuda.synchronize()
        x_cpu = x.cpu()
        ref, idx, _ = PA.check_routing(x_cpu, l_cpu, w.top_k, w.eps, w.routed_scale, rt)
        PA.check_dispatch(idx, w.n_experts, rt)
        toks = np.arange(N) if N <= 64 else np.random.default_rng(r).choice(N, 48, replace=False)
        PA.check_outputs(x_cpu, l_cpu, w.top_k, w.eps, w.routed_scale, o, idx, toks, w.dtype)
        # the same tokens through one context holding every expert
        o1 = single(x)
        torch.cuda.synchronize()
        same = (single.debug_routing(N)["idx"] == rt["idx"]).all(1)
        a, b = o1.double()[same], o.double()[same]
        ulp = 2.0 ** -23 if w.dtype == "f32" else 2.0 ** -7   # one unit of the storage type
        excess = ((a - b).abs() - ulp * torch.maximum(a.abs(), b.abs())).max().item()
        assert excess <= 1e-6, (r, excess)
    for s in shards:
        s.close()
    single.close()


def test_rank_with_nothing_to_compute():
    """A bias that sends every token to the first experts leaves the other
    ranks without rows to compute; their forwards still combine correctly."""
    w = W.DECODE.scaled(n_tokens=16)
    layer = W.make_layer(w, 0, "cuda")
    layer["bias"] = torch.full_like(layer["bias"], -1.0)
    layer["bias"][:4] = 1.0
    xs = [W.make_x(w, "cuda", seed=90 + r) for r in range(4)]
    outs = [torch.empty_like(x) for x in xs]
    shards = _shards(w, layer, 4, w.n_tokens)
    ep.emulate_ep_forward(shards, xs, outs)
    torch.cuda.synchronize()
    l_cpu = PA.to_cpu_layer(layer)
    for s, x, o in zip(shards, xs, outs):
        assert s.status() == 0
        rt = s.debug_routing(w.n_tokens)
        idx = rt["idx"].cpu().numpy()
        assert set(np.unique(idx)) == {0, 1, 2, 3}
        PA.check_outputs(x.cpu(), l_cpu, w.top_k, w.eps, w.routed_scale, o, idx,
                         np.arange(w.n_tokens), w.dtype)
    for s in shards:
        s.close()


def test_receive_capacity_is_enforced():
    w = W.DECODE.scaled(n_tokens=8)
    layer = W.make_layer(w, 0, "cuda")
    loc = dict(layer, w_gate_up=layer["w_gate_up"][:8], w_down=layer["w_down"][:8])
    s = ep.EpShard(loc, w.n_experts, 0, w.top_k, max_tokens=8, max_recv_rows=64)
    with pytest.raises(Exception):
        s.experts(np.full(8, 9, np.int32))     # 72 rows > 64
    s.close()
