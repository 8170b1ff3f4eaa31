"""Expert parallelism for the sigmoid-bias top-k MoE block: the E experts are
split over W ranks (one process per GPU), E/W contiguous experts per rank.

"LFM2.5-24B-A2B: Biased Routing, Short Convolutions and Ten KV Caches"
(flozi.net, English page), section "The router has two different scores":
once experts are spread over devices, dispatch, token regrouping and uneven
expert loads decide the cost, and expert parallelism is how such a layer is
deployed at scale. The page gives no implementation; this is one.

A forward on every rank (ep_forward):
  1. moe_ep_dispatch: the rank's own tokens are routed over all E experts and
     their normalised rows grouped by expert into the send buffer; the
     per-expert row counts come back to the host;
  2. all_gather of the counts, so every rank knows every rank's counts;
  3. exchange_plan (pure host logic): one message per (peer, expert) with
     rows, in expert order; the receiver lays its rows out grouped by local
     expert, source-rank order within an expert;
  4. exchange of the rows (grouped point-to-point send/recv: NCCL on GPUs,
     gloo on CPU; a rank's rows for itself are copied locally);
  5. moe_ep_experts: the local experts' two contractions on the received rows;
  6. the mirror exchange returns each output row to the rank and position of
     its input row;
  7. moe_ep_combine: out = x + sum_j w_j y_j in slot order.
Per rank the data path is two all-to-all-v exchanges of N*k rows of d values.
No kernel reads another GPU's memory.
"""
from __future__ import annotations

import ctypes
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

Msg = Tuple[int, int, int, int]   # (peer, expert, first row, rows)


def exchange_plan(all_counts, rank: int, n_local: int) -> Dict:
    """Messages of one rank for the row exchange.

    all_counts: [W][E] per-expert row counts of every rank's dispatch (rank
    q's rows of expert e are rows offsets_q[e] .. offsets_q[e+1]-1 of its
    send buffer, offsets_q the exclusive prefix of all_counts[q]).
    Returns dict(sends, recvs, local_counts):
      sends: (peer, expert, first row in my send buffer, rows) for every
        expert of every peer's block that I have rows for, peer-major then
        expert order;
      recvs: (peer, expert, first row in my receive buffer, rows): my
        receive buffer holds local expert 0's rows from rank 0, 1, ..., then
        local expert 1's, ...;
      local_counts: [n_local] rows per local expert.
    Between any two ranks the messages go in ascending expert order on both
    sides, so point-to-point messages match in the order they are posted.
    Empty messages are left out on both sides."""
    C = np.asarray(all_counts, dtype=np.int64)
    W, E = C.shape
    if E != W * n_local:
        raise ValueError(f"{E} experts do not split into {W} blocks of {n_local}")
    off = np.concatenate([[0], np.cumsum(C[rank])])
    sends: List[Msg] = []
    for q in range(W):
        for e in range(q * n_local, (q + 1) * n_local):
            if C[rank, e]:
                sends.append((q, e, int(off[e]), int(C[rank, e])))
    mine = C[:, rank * n_local:(rank + 1) * n_local]          # [W][n_local]
    recvs: List[Msg] = []
    pos = 0
    for el in range(n_local):
        for s in range(W):
            n = int(mine[s, el])
            if n:
                recvs.append((s, rank * n_local + el, pos, n))
            pos += n
    return {"sends": sends, "recvs": recvs, "local_counts": mine.sum(0).astype(np.int32)}


def return_plan(plan: Dict) -> Dict:
    """The mirror exchange: each received row's output goes back to where the
    row came from (sends and recvs swap roles)."""
    return {"sends": plan["recvs"], "recvs": plan["sends"], "local_counts": plan["local_counts"]}


def exchange(sends: Sequence[Msg], recvs: Sequence[Msg], send_buf, recv_buf, rank: int,
             group=None) -> None:
    """Moves rows send_buf[first:first+rows] to the peers' recv_buf as the
    plan lists them: messages to this rank itself are local copies (paired
    in order), the rest one batch of point-to-point sends and receives
    through torch.distributed (NCCL for device buffers, gloo for host)."""
    import torch.distributed as dist
    self_s = [m for m in sends if m[0] == rank]
    self_r = [m for m in recvs if m[0] == rank]
    if len(self_s) != len(self_r):
        raise RuntimeError("plan mismatch between this rank's sends and receives to itself")
    for (_, es, a, n), (_, er, b, m) in zip(self_s, self_r):
        if es != er or n != m:
            raise RuntimeError("plan mismatch between this rank's sends and receives to itself")
        recv_buf[b:b + m].copy_(send_buf[a:a + n])
    ops = [dist.P2POp(dist.isend, send_buf[a:a + n], p, group) for p, _, a, n in sends if p != rank]
    ops += [dist.P2POp(dist.irecv, recv_buf[b:b + n], p, group) for p, _, b, n in recvs if p != rank]
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()


def gather_counts(counts, group=None, device=None) -> np.ndarray:
    """[W][E] counts of every rank (all_gather of each rank's [E] counts)."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    t = torch.as_tensor(np.asarray(counts, dtype=np.int64), device=device)
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t, group=group)
    return torch.stack(parts).cpu().numpy()


# ----------------------------------------------------------------- C-ABI shard
class _DeviceArray:
    """A device address seen as a typed array (for torch.as_tensor)."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"data": (ptr, False), "shape": tuple(shape),
                                         "typestr": typestr, "strides": None, "version": 3}


def _view(ptr: int, rows: int, cols: int, dtype, device):
    import torch
    if dtype == torch.bfloat16:
        t = torch.as_tensor(_DeviceArray(ptr, (rows, cols), "<i2"), device=device)
        return t.view(torch.bfloat16)
    return torch.as_tensor(_DeviceArray(ptr, (rows, cols), "<f4"), device=device)


class EpShard:
    """One rank's part of an expert-parallel layer (moe_ep_* in include/moe.h).

    layer: dict with the WHOLE router (norm_gain [d], router_w [E,d], bias
    [E], f32) and the LOCAL experts only: w_gate_up [n_local,2I,d], w_down
    [n_local,d,I] (bf16 or f32), on this rank's CUDA device."""

    def __init__(self, layer: Dict, n_experts: int, expert_first: int, top_k: int,
                 eps: float = 1e-6, routed_scale: float = 1.0, max_tokens: int = 1024,
                 max_recv_rows: Optional[int] = None, world: int = 1):
        import torch
        from . import MoeWeights, MOE_BF16, MOE_F32, _check, lib
        wgu = layer["w_gate_up"]
        n_local, twoI, d = wgu.shape
        if wgu.dtype not in (torch.bfloat16, torch.float32):
            raise TypeError("expert parallelism takes bf16 or f32 experts")
        self.d, self.E, self.I, self.k = d, n_experts, twoI // 2, top_k
        self.n_local, self.expert_first = n_local, expert_first
        self.dtype, self.device = wgu.dtype, wgu.device
        self.max_tokens = max_tokens
        self.max_recv_rows = max_recv_rows or world * max_tokens * top_k
        names = ["norm_gain", "router_w", "bias", "w_gate_up", "w_down"]
        self._keep = {n: layer[n].contiguous() for n in names}
        k = self._keep
        dt = MOE_BF16 if wgu.dtype == torch.bfloat16 else MOE_F32
        self._w = MoeWeights(dt, k["norm_gain"].data_ptr(), k["router_w"].data_ptr(),
                             k["bias"].data_ptr(), k["w_gate_up"].data_ptr(),
                             k["w_down"].data_ptr(), routed_scale, None, None)
        L = lib()
        h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            _check(L.moe_ep_create(d, n_experts, self.I, top_k, eps, ctypes.byref(self._w),
                                   max_tokens, expert_first, n_local, self.max_recv_rows,
                                   ctypes.byref(h)), "moe_ep_create")
        self._h = h
        p = [ctypes.c_void_p() for _ in range(4)]
        _check(L.moe_ep_buffers(h, *[ctypes.byref(x) for x in p]), "moe_ep_buffers")
        R, C = max_tokens * top_k, self.max_recv_rows
        self.send_rows = _view(p[0].value, R, d, self.dtype, self.device)
        self.recv_rows = _view(p[1].value, C, d, self.dtype, self.device)
        self.send_y = _view(p[2].value, C, d, self.dtype, self.device)
        self.recv_y = _view(p[3].value, R, d, self.dtype, self.device)

    def dispatch(self, x, stream=None) -> np.ndarray:
        from . import _check, _stream_ptr, lib
        counts = np.zeros(self.E, np.int32)
        _check(lib().moe_ep_dispatch(self._h, x.data_ptr(), x.shape[0], counts.ctypes.data,
                                     _stream_ptr(stream)), "moe_ep_dispatch")
        return counts

    def experts(self, local_counts, stream=None) -> None:
        from . import _check, _stream_ptr, lib
        lc = np.ascontiguousarray(np.asarray(local_counts, dtype=np.int32))
        if lc.shape != (self.n_local,):
            raise ValueError(f"local_counts must have {self.n_local} entries")
        _check(lib().moe_ep_experts(self._h, lc.ctypes.data, _stream_ptr(stream)),
               "moe_ep_experts")

    def combine(self, x, out, stream=None):
        from . import _check, _stream_ptr, lib
        _check(lib().moe_ep_combine(self._h, x.data_ptr(), out.data_ptr(), _stream_ptr(stream)),
               "moe_ep_combine")
        return out

    def debug_routing(self, n_tokens: int, stream=None):
        import torch
        from . import _check, _stream_ptr, lib
        dev = self.device
        r = {"idx": torch.empty(n_tokens, self.k, dtype=torch.int32, device=dev),
             "w": torch.empty(n_tokens, self.k, dtype=torch.float32, device=dev),
             "perm": torch.empty(n_tokens * self.k, dtype=torch.int32, device=dev),
             "offsets": torch.empty(self.E + 1, dtype=torch.int32, device=dev)}
        _check(lib().moe_ep_debug_routing(self._h, r["idx"].data_ptr(), r["w"].data_ptr(),
                                          r["perm"].data_ptr(), r["offsets"].data_ptr(),
                                          _stream_ptr(stream)), "moe_ep_debug_routing")
        return r

    def status(self) -> int:
        from . import lib
        return lib().moe_ep_status(self._h)

    def close(self):
        from . import _check, lib
        if getattr(self, "_h", None):
            rc = lib().moe_ep_destroy(self._h)
            self._h = None
            _check(rc, "moe_ep_destroy")

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def ep_forward(shard, x, out=None, group=None):
    """One expert-parallel forward on this rank (all ranks call it together)."""
    import torch
    import torch.distributed as dist
    rank = dist.get_rank(group)
    counts = shard.dispatch(x)
    allc = gather_counts(counts, group, device=x.device)
    plan = exchange_plan(allc, rank, shard.n_local)
    exchange(plan["sends"], plan["recvs"], shard.send_rows, shard.recv_rows, rank, group)
    shard.experts(plan["local_counts"])
    back = return_plan(plan)
    exchange(back["sends"], back["recvs"], shard.send_y, shard.recv_y, rank, group)
    if out is None:
        out = torch.empty_like(x)
    return shard.combine(x, out)


def emulate_ep_forward(shards: Sequence["EpShard"], xs: Sequence, outs: Sequence) -> None:
    """All W ranks of one expert-parallel forward run in turn in this process
    (on one device): the same plans, with the exchanges done as local copies
    between the shards' buffers. For testing the shards' compute where fewer
    GPUs than ranks are available; no kernel waits on another."""
    W = len(shards)
    counts = np.stack([s.dispatch(x) for s, x in zip(shards, xs)])
    plans = [exchange_plan(counts, r, shards[r].n_local) for r in range(W)]
    _local_exchange(plans, [s.send_rows for s in shards], [s.recv_rows for s in shards])
    for s, p in zip(shards, plans):
        s.experts(p["local_counts"])
    backs = [return_plan(p) for p in plans]
    _local_exchange(backs, [s.send_y for s in shards], [s.recv_y for s in shards])
    for s, x, o in zip(shards, xs, outs):
        s.combine(x, o)


def _local_exchange(plans, send_bufs, recv_bufs) -> None:
    """Carries out every rank's plan at once: rank r's i-th send to peer q is
    paired with q's i-th receive from r."""
    W = len(plans)
    for r in range(W):
        for q in range(W):
            snd = [m for m in plans[r]["sends"] if m[0] == q]
            rcv = [m for m in plans[q]["recvs"] if m[0] == r]
            if len(snd) != len(rcv):
                raise RuntimeError(f"plans of ranks {r} and {q} do not match")
            for (_, e1, a, n), (_, e2, b, m) in zip(snd, rcv):
                if e1 != e2 or n != m:
                    raise RuntimeError(f"plans of ranks {r} and {q} do not match")
                recv_bufs[q][b:b + m].copy_(send_bufs[r][a:a + n])
