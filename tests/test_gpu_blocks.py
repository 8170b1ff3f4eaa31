"""Parity of the dense feed-forward block and the short-convolution block
(include/block.h, through the C ABI) with the fp64 oracle. Needs an sm_100 GPU.

Tolerances as for the MoE block's bf16 layers: per token ||o - ref|| /
||ref|| <= 1e-2, and the block's own contribution o - x within 1e-2 of
||ref - x|| plus the bf16 rounding of the stored output (2^-8 ||ref||), the
GPU rounding the normalised rows and the intermediate streams (act; a, y)
to bf16 once each."""
import numpy as np
import pytest
import torch

import oracle
from sigmoid_bias_top_b200 import workloads as W
from sigmoid_bias_top_b200.blocks import ConvBlock, DenseBlock

pytestmark = pytest.mark.gpu

TOL, DELTA_TOL, OUT_ROUND = 1e-2, 1e-2, 2.0 ** -8


def check(o_gpu, ref, x):
    """o_gpu, x: [n, d] tensors; ref: [n, d] f64 numpy."""
    o = o_gpu.double().cpu().numpy().reshape(ref.shape)
    xd = x.double().cpu().numpy().reshape(ref.shape)
    err = np.linalg.norm(o - ref, axis=1) / np.linalg.norm(ref, axis=1)
    assert err.max() <= TOL, err.max()
    dn = np.maximum(np.linalg.norm(ref - xd, axis=1), 1e-30)
    derr = np.linalg.norm((o - xd) - (ref - xd), axis=1) / dn
    allowed = DELTA_TOL + OUT_ROUND * np.linalg.norm(ref, axis=1) / dn
    assert np.all(derr <= allowed), (derr / allowed).max()
    return float(err.max()), float(derr.max())


def cpu(layer):
    return {k: v.detach().cpu() for k, v in layer.items()}


@pytest.fixture(params=["split", "unsplit"])
def split_mode(request, monkeypatch):
    """Small batches split K across the GPU (partial sums, then a reduce
    launch); MOE_BLOCK_SPLIT=0 at create keeps every GEMM whole. Both paths
    must give the same result."""
    if request.param == "unsplit":
        monkeypatch.setenv("MOE_BLOCK_SPLIT", "0")
    else:
        monkeypatch.delenv("MOE_BLOCK_SPLIT", raising=False)
    return request.param


# ------------------------------------------------------------------ dense
@pytest.mark.parametrize("n,d,I", [(300, 256, 320), (1, 128, 64), (513, 192, 448)])
def test_dense_ragged(n, d, I, split_mode):
    w = W.DENSE_PREFILL.scaled(n_seqs=n, seq_len=1, d=d, d_ff=I, w_std=0.06)
    layer = W.make_block_layer(w, "cuda")
    x = W.make_block_x(w, "cuda")
    blk = DenseBlock(layer, w.eps, max_tokens=n)
    out = blk(x)
    torch.cuda.synchronize()
    assert blk.status() == 0
    check(out, oracle.dense_ffn(x.cpu(), cpu(layer), w.eps), x)
    blk.close()


@pytest.mark.parametrize("name", ["dense_decode", "dense_prefill"])
def test_dense_full_size_sampled(name):
    w = W.BLOCK_WORKLOADS[name]
    layer = W.make_block_layer(w, "cuda")
    x = W.make_block_x(w, "cuda")
    blk = DenseBlock(layer, w.eps, max_tokens=w.n_tokens)
    out = blk(x)
    torch.cuda.synchronize()
    assert blk.status() == 0
    toks = np.arange(w.n_tokens) if w.n_tokens <= 64 else np.unique(np.concatenate(
        [[0, w.n_tokens - 1], np.random.default_rng(1).choice(w.n_tokens, 96, replace=False)]))
    idx = torch.as_tensor(toks)
    ref = oracle.dense_ffn(x.cpu()[idx], cpu(layer), w.eps)
    check(out[idx.cuda()], ref, x[idx.cuda()])
    blk.close()


def test_dense_in_place_and_deterministic(split_mode):
    w = W.DENSE_PREFILL.scaled(n_seqs=260, seq_len=1, d=256, d_ff=256)
    layer = W.make_block_layer(w, "cuda")
    x = W.make_block_x(w, "cuda")
    blk = DenseBlock(layer, w.eps, max_tokens=260)
    a = blk(x)
    b = blk(x)
    y = x.clone()
    blk(y, y)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(a, y)
    blk.close()


# ------------------------------------------------------------------ conv
def conv_ref(x, layer, eps, state=None):
    return oracle.shortconv(x.cpu(), cpu(layer), eps,
                            state_in=None if state is None else state.cpu().double().numpy())


@pytest.mark.parametrize("B,T,d", [(3, 300, 256), (1, 1, 128), (2, 7, 192), (5, 130, 64)])
def test_conv_ragged(B, T, d, split_mode):
    """Sequences that cross the GEMM's 256-row token tiles, ragged tails, T < 3."""
    w = W.CONV_PREFILL.scaled(n_seqs=B, seq_len=T, d=d, w_std=0.06)
    layer = W.make_block_layer(w, "cuda")
    x = W.make_block_x(w, "cuda")
    blk = ConvBlock(layer, w.eps, max_tokens=B * T)
    st_out = torch.full((B, 2, d), float("nan"), device="cuda")
    out = blk(x, state_out=st_out)
    torch.cuda.synchronize()
    assert blk.status() == 0
    ref, ref_state = conv_ref(x, layer, w.eps)
    check(out.reshape(-1, d), ref.reshape(-1, d), x.reshape(-1, d))
    # the carried a values are the GPU's bf16 a: within bf16 rounding of the oracle's
    np.testing.assert_allclose(st_out.double().cpu().numpy(), ref_state, rtol=2e-2, atol=2e-2)


def test_conv_carried_state_and_decode_steps(split_mode):
    """Prefill T1 positions, then T2 more with the state carried, then three
    decode steps (T = 1), against the oracle on the whole sequences."""
    B, d = 3, 256
    w = W.CONV_PREFILL.scaled(n_seqs=B, seq_len=40, d=d, w_std=0.06)
    layer = W.make_block_layer(w, "cuda")
    x = W.make_block_x(w, "cuda")
    blk = ConvBlock(layer, w.eps, max_tokens=B * 40)
    st = torch.zeros(B, 2, d, device="cuda")
    parts = []
    for t0, t1 in ((0, 29), (29, 37), (37, 38), (38, 39), (39, 40)):
        xs = x[:, t0:t1].contiguous()
        parts.append(blk(xs, state_in=st, state_out=st))   # state updated in place
    torch.cuda.synchronize()
    assert blk.status() == 0
    out = torch.cat(parts, 1)
    ref, _ = conv_ref(x, layer, w.eps)
    check(out.reshape(-1, d), ref.reshape(-1, d), x.reshape(-1, d))


def test_conv_decode_with_given_state():
    w = W.CONV_DECODE
    layer = W.make_block_layer(w, "cuda")
    x = W.make_block_x(w, "cuda")
    st = W.make_conv_state(w, "cuda")
    blk = ConvBlock(layer, w.eps, max_tokens=w.n_tokens)
    st_out = torch.empty_like(st)
    out = blk(x, state_in=st, state_out=st_out)
    torch.cuda.synchronize()
    assert blk.status() == 0
    ref, ref_state = conv_ref(x, layer, w.eps, state=st)
    check(out.reshape(-1, w.d), ref.reshape(-1, w.d), x.reshape(-1, w.d))
    assert torch.equal(st_out[:, 0], st[:, 1])        # the old position -1 moves to -2
    np.testing.assert_allclose(st_out[:, 1].double().cpu().numpy(), ref_state[:, 1],
                               rtol=2e-2, atol=2e-2)


def test_conv_prefill_full_size_windows():
    """The 4 x 2048-position prefill, checked on three windows of every
    sequence: the start, the middle and the end. An output at position t
    depends on x at t, t-1, t-2 only, and the a of a position on that
    position's x only, so each window's expected values are the oracle on the
    window with the a of the two positions before it as the state."""
    w = W.CONV_PREFILL
    layer = W.make_block_layer(w, "cuda")
    x = W.make_block_x(w, "cuda")
    blk = ConvBlock(layer, w.eps, max_tokens=w.n_tokens)
    out = blk(x)
    torch.cuda.synchronize()
    assert blk.status() == 0
    for s in (0, 1000, w.seq_len - 48):
        state = None
        if s >= 2:
            _, state = conv_ref(x[:, s - 2:s].contiguous(), layer, w.eps)
            state = torch.from_numpy(state)
        ref, _ = conv_ref(x[:, s:s + 48].contiguous(), layer, w.eps, state=state)
        check(out[:, s:s + 48].reshape(-1, w.d), ref.reshape(-1, w.d),
              x[:, s:s + 48].reshape(-1, w.d))
    blk.close()


def test_conv_in_place_and_deterministic(split_mode):
    w = W.CONV_PREFILL.scaled(n_seqs=2, seq_len=300, d=256)
    layer = W.make_block_layer(w, "cuda")
    x = W.make_block_x(w, "cuda")
    blk = ConvBlock(layer, w.eps, max_tokens=600)
    a = blk(x)
    b = blk(x)
    y = x.clone()
    blk(y, y)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(a, y)
    blk.close()
