"""Comparison of the CUDA path with the fp64 oracle (helpers for the GPU tests).

Rules (the tolerances the tests assert):
  * the selected set is exact for every token whose margin c_(k) - c_(k+1)
    between the last selected and the best unselected biased score exceeds
    1e-3 in the oracle, and so is the slot order, except between two selected
    experts whose biased scores are within 1e-5 of each other (equal keys under
    fp32 rounding), where the GPU's order must still be descending within 1e-5;
  * for the other (near-tie) tokens, the GPU's set is accepted if every expert
    it selected has c >= c_(k) - 1e-3 in the oracle, and that token's output
    is compared with the oracle recomputed on the GPU's selection;
  * the dispatch permutation and offsets equal the oracle's counting sort of
    the GPU's own selection, exactly;
  * mixture weights agree to 1e-5 relative (fp32 sigmoid vs fp64);
  * outputs: per token ||o_gpu - o_ref|| / ||o_ref|| <= 1e-2 for bf16 storage
    (FP8_BLOCK layers store x and out as bf16 too), 1e-5 for fp32 storage;
  * the MoE part alone is bounded too, since the residual x dominates ||out||
    (on the decode step the MoE part is under a fifth of it, so the bound on
    out alone would admit a 5% error in the part the kernels compute): per
    token ||(o_gpu - x) - (o_ref - x)|| / ||o_ref - x|| <= DELTA_TOL + u
    ||o_ref|| / ||o_ref - x||, where u is the rounding of the stored out
    (2^-8 of |out| per element for bf16, 2^-24 for fp32), which the second
    term admits. DELTA_TOL is 1e-2 for bf16 layers (the GPU rounds the
    normalised rows, SiLU(gate)*up and the expert outputs to bf16, 2^-9
    relative each), 2e-2 for FP8_BLOCK layers (the oracle applies the same
    e4m3 quantisation, so what remains is fp32 summation order, the bf16
    rounding of the expert outputs and the rare e4m3 code that rounds the
    other way because the two sides' fp32 inputs differ in the last bits: one
    code step is 1/16 of one value out of 128) and 1e-4 for fp32 layers;
  * near ties are rare: the number of tokens whose margin is at most 1e-3 is
    bounded by NEAR_FRAC of the batch plus NEAR_SLACK (the workloads have
    4-10%), so a margin computed too small cannot move most tokens out of the
    exact checks.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

MARGIN = 1e-3
ORDER_GAP = 1e-5   # selected experts closer than this may swap slots under fp32 rounding
TOL = {"bf16": 1e-2, "f32": 1e-5, "fp8": 1e-2}
DELTA_TOL = {"bf16": 1e-2, "fp8": 2e-2, "f32": 1e-4}
OUT_ROUND = {"bf16": 2.0 ** -8, "fp8": 2.0 ** -8, "f32": 2.0 ** -24}
NEAR_FRAC, NEAR_SLACK = 0.2, 2
W_RTOL = 1e-5


def to_cpu_layer(layer):
    return {k: v.detach().cpu() for k, v in layer.items()}


def check_routing(x_cpu, layer_cpu, k, eps, scale, r_gpu):
    """Returns the oracle routing and the GPU idx (numpy); asserts the rules."""
    ref = oracle.route(x_cpu, layer_cpu, k, eps, scale)
    idx = r_gpu["idx"].cpu().numpy()
    w = r_gpu["w"].cpu().numpy().astype(np.float64)
    N = idx.shape[0]
    b = layer_cpu["bias"].double().numpy()
    c = ref["s"] + b[None, :]
    clear = ref["margin"] > MARGIN
    set_bad = np.where(clear & np.any(np.sort(idx, 1) != np.sort(ref["idx"], 1), axis=1))[0]
    assert set_bad.size == 0, (
        f"{set_bad.size} tokens with margin > {MARGIN} select another set; first: "
        + "; ".join(f"t={t} gpu={idx[t].tolist()} ref={ref['idx'][t].tolist()} "
                    f"margin={ref['margin'][t]:.3e}" for t in set_bad[:3]))
    c_ref_sel = np.take_along_axis(c, ref["idx"].astype(np.int64), 1)
    gap = -np.diff(c_ref_sel, axis=1)                    # >= 0, oracle slot order
    strict = clear & (gap.min(1) > ORDER_GAP if k > 1 else np.ones(N, bool))
    ord_bad = np.where(strict & np.any(idx != ref["idx"], axis=1))[0]
    assert ord_bad.size == 0, (
        f"{ord_bad.size} tokens differ in slot order; first: "
        + "; ".join(f"t={t} gpu={idx[t].tolist()} ref={ref['idx'][t].tolist()} "
                    f"gaps={gap[t].tolist()}" for t in ord_bad[:3]))
    c_gpu_sel = np.take_along_axis(c, idx.astype(np.int64), 1)
    assert np.all(np.diff(c_gpu_sel, axis=1) <= ORDER_GAP), "GPU slots not in descending c"
    # near ties: every GPU-selected expert is within MARGIN of the k-th best
    n_near = int((~clear).sum())
    assert n_near <= NEAR_FRAC * N + NEAR_SLACK, (
        f"{n_near} of {N} tokens have margin <= {MARGIN}: more near ties than the inputs allow")
    ck = np.take_along_axis(c, ref["idx"][:, -1:].astype(np.int64), 1)[:, 0]
    for t in np.where(~clear)[0]:
        sel = idx[t]
        assert len(set(sel.tolist())) == k and sel.min() >= 0, (t, sel)
        assert np.all(c[t, sel] >= ck[t] - MARGIN), (t, sel, c[t, sel], ck[t])
    # weights from the unbiased scores of the GPU's own selection
    s_sel = np.take_along_axis(ref["s"], idx.astype(np.int64), 1)
    w_ref = scale * s_sel / (s_sel.sum(1, keepdims=True) + eps)
    np.testing.assert_allclose(w, w_ref, rtol=W_RTOL, atol=1e-7)
    return ref, idx, n_near


def check_dispatch(idx, n_experts, r_gpu):
    d = oracle.dispatch(idx, n_experts)
    np.testing.assert_array_equal(r_gpu["offsets"].cpu().numpy(), d["offsets"])
    np.testing.assert_array_equal(r_gpu["perm"].cpu().numpy(), d["perm"])
    return d


def check_outputs(x_cpu, layer_cpu, k, eps, scale, out_gpu, idx, tokens, dtype):
    tokens = np.asarray(tokens, dtype=np.int64)
    ref = oracle.forward(x_cpu, layer_cpu, k, eps, scale, tokens=tokens, forced=idx[tokens])
    o = out_gpu[torch.as_tensor(tokens, device=out_gpu.device)].double().cpu().numpy()
    err = np.linalg.norm(o - ref["out"], axis=1) / np.linalg.norm(ref["out"], axis=1)
    x = x_cpu[torch.as_tensor(tokens)].double().numpy()
    delta_err = (np.linalg.norm((o - x) - (ref["out"] - x), axis=1)
                 / np.maximum(np.linalg.norm(ref["out"] - x, axis=1), 1e-30))
    tol = TOL[dtype]
    worst = int(np.argmax(err))
    assert err.max() <= tol, (f"max rel-L2 {err.max():.3e} > {tol} at token {tokens[worst]}; "
                              f"MoE-delta rel err {delta_err[worst]:.3e}")
    dn = np.maximum(np.linalg.norm(ref["out"] - x, axis=1), 1e-30)
    allowed = DELTA_TOL[dtype] + OUT_ROUND[dtype] * np.linalg.norm(ref["out"], axis=1) / dn
    wd = int(np.argmax(delta_err / allowed))
    assert np.all(delta_err <= allowed), (
        f"MoE-delta rel-L2 {delta_err[wd]:.3e} > {allowed[wd]:.3e} at token {tokens[wd]}")
    return float(err.max()), float(delta_err.max())


def sample_tokens(N, idx, offsets, n_random=192, seed=0):
    """First/last tokens, tokens of the least-loaded non-empty experts, and a
    seeded random sample."""
    rng = np.random.default_rng(seed)
    pick = {0, N - 1}
    counts = np.diff(offsets)
    for e in np.argsort(counts):
        if counts[e] == 0:
            continue
        hits = np.where((idx == e).any(1))[0]
        pick.update(hits[:4].tolist())
        if len(pick) > 40:
            break
    pick.update(rng.choice(N, size=min(n_random, N), replace=False).tolist())
    return np.array(sorted(pick), dtype=np.int64)
