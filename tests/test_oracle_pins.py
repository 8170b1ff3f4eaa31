"""The oracle against its pins, and every planted mistake caught by a pin."""
import numpy as np
import pytest
import torch

import oracle
from tests import oracle_pins as P
from sigmoid_bias_top_b200 import workloads as W


@pytest.mark.parametrize("pin", P.PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(0)


@pytest.mark.parametrize("name", [n for n in oracle.MUTATIONS if n != "none"])
def test_planted_mistake_is_caught(name):
    """Each planted mistake in the oracle fails at least one pin."""
    mut = oracle.MUTATIONS[name]
    caught = []
    for pin in P.PINS:
        try:
            pin(mut)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"planted mistake {name!r} passes every pin"


def test_dispatch_is_stable_counting_sort():
    """perm lists assignments expert by expert, ascending token within an
    expert: the same as Python's stable sort of assignment ids by expert."""
    layer = P.rand_layer(10, 16, 4, seed=7, bias_scale=0.6)
    r = oracle.route(P.rand_x(97, 16, 7), layer, k=3, eps=P.EPS)
    dsp = oracle.dispatch(r["idx"], 10)
    flat = r["idx"].reshape(-1)
    want = sorted(range(flat.size), key=lambda a: flat[a])
    np.testing.assert_array_equal(dsp["perm"], np.array(want, np.int32))
    np.testing.assert_array_equal(dsp["counts"], np.bincount(flat, minlength=10))
    np.testing.assert_array_equal(dsp["offsets"], np.concatenate([[0], np.cumsum(dsp["counts"])]))


def test_dispatch_empty_and_all_one_expert():
    d0 = oracle.dispatch(np.zeros((0, 4), np.int32), 8)
    assert d0["counts"].sum() == 0 and d0["perm"].size == 0
    idx = np.full((5, 1), 3, np.int32)
    d1 = oracle.dispatch(idx, 8)
    assert d1["counts"].tolist() == [0, 0, 0, 5, 0, 0, 0, 0]
    assert d1["perm"].tolist() == [0, 1, 2, 3, 4]


def test_wrong_models_differ_beyond_tolerance():
    """Softmax in place of sigmoid, and the biased scores used as weights, are
    different models: their outputs differ from the oracle's far beyond the
    1e-5 (fp32) parity tolerance on the tiny f32 workload."""
    w = W.TINY_F32
    x, layers = W.make_inputs(w)
    ref = oracle.forward(x, layers[0], w.top_k, w.eps)["out"]
    for name in ("softmax", "biased_weights"):
        o = oracle.forward(x, layers[0], w.top_k, w.eps, mutation=oracle.MUTATIONS[name])["out"]
        rel = np.linalg.norm(o - ref, axis=1) / np.linalg.norm(ref, axis=1)
        assert rel.max() > 1e-2, (name, rel.max())


def test_bf16_values_widen_exactly():
    """bf16 storage is read as the exact float it encodes."""
    x = torch.tensor([[1.0, -2.5, 3.140625, 0.0078125]], dtype=torch.bfloat16)
    gain = torch.ones(4)
    a = oracle.rmsnorm(x, gain, 0.0)
    b = oracle.rmsnorm(x.float(), gain, 0.0)
    assert np.array_equal(a, b)
