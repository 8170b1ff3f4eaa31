"""Expert parallelism on the CPU: the exchange plan's invariants, and whole
expert-parallel forwards on gloo ranks (world size 2 and 8) whose shards are
stood in for by the fp64 oracle, moved by the same plan and exchange code the
GPU ranks use, against the oracle's single-process forward."""
import os
import socket

import numpy as np
import pytest
import torch

from sigmoid_bias_top_b200 import ep


def _random_counts(W, E, seed, zero_frac=0.3):
    rng = np.random.default_rng(seed)
    c = rng.integers(0, 40, size=(W, E))
    c[rng.random((W, E)) < zero_frac] = 0
    return c


@pytest.mark.parametrize("W,n_local", [(1, 4), (2, 8), (8, 8), (4, 1)])
def test_exchange_plan_matches_across_ranks(W, n_local):
    """Every row of every rank is sent exactly once, to the rank owning its
    expert; each pair's sends and receives list the same experts and sizes in
    the same order; receive buffers are filled expert-major without gaps."""
    E = W * n_local
    C = _random_counts(W, E, seed=W * 100 + n_local)
    plans = [ep.exchange_plan(C, r, n_local) for r in range(W)]
    for r in range(W):
        sent = np.zeros(C[r].sum(), int)
        for q, e, a, n in plans[r]["sends"]:
            assert q == e // n_local and n == C[r, e]
            sent[a:a + n] += 1
        assert (sent == 1).all()
        for q in range(W):
            snd = [(e, n) for p, e, _, n in plans[r]["sends"] if p == q]
            rcv = [(e, n) for p, e, _, n in plans[q]["recvs"] if p == r]
            assert snd == rcv
        lc = plans[r]["local_counts"]
        assert lc.tolist() == C[:, r * n_local:(r + 1) * n_local].sum(0).tolist()
        pos = 0
        for p, e, b, n in plans[r]["recvs"]:      # contiguous, expert-major, rank order
            assert b == pos
            pos += n
        assert pos == lc.sum()
        keys = [(e, p) for p, e, _, _ in plans[r]["recvs"]]
        assert keys == sorted(keys)
    back = ep.return_plan(plans[0])
    assert back["sends"] == plans[0]["recvs"] and back["recvs"] == plans[0]["sends"]


def test_exchange_plan_rejects_uneven_split():
    with pytest.raises(ValueError):
        ep.exchange_plan(np.zeros((3, 8), int), 0, 2)


# ------------------------------------------------------------- gloo ranks
E_TOTAL, D, I, K, TOKENS = 16, 32, 16, 4, 24


def _layer(seed=3):
    g = torch.Generator().manual_seed(seed)
    return {
        "norm_gain": (1 + 0.1 * torch.randn(D, generator=g)).float(),
        "router_w": (torch.randn(E_TOTAL, D, generator=g) / D ** 0.5).float(),
        # a skewed bias: some experts get many rows, some none
        "bias": torch.linspace(0.4, -0.4, E_TOTAL).float(),
        "w_gate_up": (torch.randn(E_TOTAL, 2 * I, D, generator=g) / D ** 0.5).float(),
        "w_down": (torch.randn(E_TOTAL, D, I, generator=g) / I ** 0.5).float(),
    }


class OracleShard:
    """A rank's shard with the oracle doing the compute (test stand-in for
    the CUDA shard): the same buffers and phases as ep.EpShard."""

    def __init__(self, layer, rank, world):
        import oracle
        self.o = oracle
        self.layer = layer
        self.n_local = E_TOTAL // world
        self.e0 = rank * self.n_local
        self.local = dict(layer, w_gate_up=layer["w_gate_up"][self.e0:self.e0 + self.n_local],
                          w_down=layer["w_down"][self.e0:self.e0 + self.n_local])
        cap = world * TOKENS * K
        self.send_rows = torch.zeros(TOKENS * K, D, dtype=torch.float64)
        self.recv_rows = torch.zeros(cap, D, dtype=torch.float64)
        self.send_y = torch.zeros(cap, D, dtype=torch.float64)
        self.recv_y = torch.zeros(TOKENS * K, D, dtype=torch.float64)

    def dispatch(self, x):
        self.r = self.o.route(x, self.layer, K, 1e-6)
        dsp = self.o.dispatch(self.r["idx"], E_TOTAL)
        self.inv = np.empty(TOKENS * K, np.int64)
        self.inv[dsp["perm"]] = np.arange(TOKENS * K)
        xn = self.o.rmsnorm(x, self.layer["norm_gain"], 1e-6)
        self.send_rows[:] = torch.from_numpy(xn[dsp["perm"] // K])
        return dsp["counts"]

    def experts(self, local_counts):
        pos = 0
        for el, n in enumerate(local_counts):
            if n:
                rows = self.recv_rows[pos:pos + n].numpy()
                self.send_y[pos:pos + n] = torch.from_numpy(self.o.expert(rows, self.local, el))
            pos += n

    def combine(self, x):
        out = x.double().numpy().copy()
        y = self.recv_y.numpy()
        for t in range(TOKENS):
            for j in range(K):
                out[t] += self.r["w"][t, j] * y[self.inv[t * K + j]]
        return out


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        layer = _layer()
        x = torch.randn(TOKENS, D, generator=torch.Generator().manual_seed(50 + rank))
        shard = OracleShard(layer, rank, world)
        counts = shard.dispatch(x)
        allc = ep.gather_counts(counts)
        plan = ep.exchange_plan(allc, rank, shard.n_local)
        ep.exchange(plan["sends"], plan["recvs"], shard.send_rows, shard.recv_rows, rank)
        shard.experts(plan["local_counts"])
        back = ep.return_plan(plan)
        ep.exchange(back["sends"], back["recvs"], shard.send_y, shard.recv_y, rank)
        out = shard.combine(x)
        ref = oracle.forward(x, layer, K, 1e-6)["out"]
        results[rank] = (float(np.abs(out - ref).max()), int(allc.sum()),
                         int((allc.sum(0) == 0).sum()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 8])
def test_ep_forward_on_gloo_ranks_matches_the_oracle(world):
    import torch.multiprocessing as mp
    mgr = mp.Manager()
    results = mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), results), nprocs=world, join=True)
    assert sorted(results.keys()) == list(range(world))
    for r, (err, total, empty) in results.items():
        assert err <= 1e-12, (r, err)
        assert total == world * TOKENS * K
    # the skewed bias leaves some experts without rows on every rank
    assert results[0][2] > 0
