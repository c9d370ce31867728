"""Pins of the oracle's backward pass against facts fixed outside it.

The backward is the chain rule through each expert's MLP.  A slip in it (a
dropped factor 2 in the squared-ReLU derivative, gate and up swapped in the
SwiGLU derivative, a missing top-k weight, a transposed weight gradient)
fails at least one of:

* exact linearity: the loss L = sum(dout * out) is linear in W2 and in the
  top-k weights, so L(p + delta) - L(p) = <dL/dp, delta> up to fp64 rounding
  for any delta;
* Euler's identity for homogeneous functions: out is homogeneous of degree
  1 in W2 and in the top-k weights, and (squared ReLU) of degree 2 in W13;
* central finite differences of the forward for x and W13;
* automatic differentiation (torch autograd, fp64, CPU) of the forward
  written from the layer's definition.
"""
import numpy as np
import pytest
import torch

import oracle

ACTS = [oracle.ACT_SWIGLU, oracle.ACT_RELU2]


def _problem(seed, act, T=5, d=6, F=4, E=3, k=2, shared=False):
    rng = np.random.default_rng(seed)
    n1 = 2 * F if act == oracle.ACT_SWIGLU else F
    x = rng.standard_normal((T, d))
    W13 = rng.standard_normal((E, n1, d)) * 0.5
    W2 = rng.standard_normal((E, d, F)) * 0.5
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    w = rng.random((T, k)) + 0.1
    dout = rng.standard_normal((T, d))
    S13 = rng.standard_normal((1, n1, d)) * 0.5 if shared else None
    S2 = rng.standard_normal((1, d, F)) * 0.5 if shared else None
    return x, W13, W2, ids, w, dout, S13, S2


def _loss(x, W13, W2, ids, w, act, dout, S13=None, S2=None):
    return float(np.sum(dout * oracle.forward_values(x, W13, W2, ids, w, act, S13, S2)))


@pytest.mark.parametrize("act", ACTS)
def test_linear_in_w2_and_topk_weights_exactly(act):
    x, W13, W2, ids, w, dout, _, _ = _problem(1, act)
    g = oracle.backward_values(x, W13, W2, ids, w, act, dout)
    rng = np.random.default_rng(7)
    L0 = _loss(x, W13, W2, ids, w, act, dout)
    dW2 = rng.standard_normal(W2.shape)
    assert _loss(x, W13, W2 + dW2, ids, w, act, dout) - L0 == pytest.approx(np.sum(g["dw2"] * dW2), rel=1e-10,
                                                                            abs=1e-10)
    dw = rng.standard_normal(w.shape)
    assert _loss(x, W13, W2, ids, w + dw, act, dout) - L0 == pytest.approx(
        np.sum(g["dtopk_weights"] * dw), rel=1e-10, abs=1e-10)


@pytest.mark.parametrize("act", ACTS)
def test_euler_identities(act):
    x, W13, W2, ids, w, dout, _, _ = _problem(2, act)
    g = oracle.backward_values(x, W13, W2, ids, w, act, dout)
    L = _loss(x, W13, W2, ids, w, act, dout)
    assert np.sum(g["dw2"] * W2) == pytest.approx(L, rel=1e-12)            # degree 1 in W2
    assert np.sum(g["dtopk_weights"] * w) == pytest.approx(L, rel=1e-12)   # degree 1 in the weights
    if act == oracle.ACT_RELU2:
        assert np.sum(g["dw13"] * W13) == pytest.approx(2.0 * L, rel=1e-12)  # degree 2 in fc1
        assert np.sum(g["dx"] * x) == pytest.approx(2.0 * L, rel=1e-12)      # and in x


@pytest.mark.parametrize("act", ACTS)
@pytest.mark.parametrize("shared", [False, True])
def test_central_finite_differences(act, shared):
    x, W13, W2, ids, w, dout, S13, S2 = _problem(3, act, shared=shared)
    g = oracle.backward_values(x, W13, W2, ids, w, act, dout, S13, S2)
    h = 1e-6

    def fd(arr, idx):
        old = arr[idx]
        arr[idx] = old + h
        lp = _loss(x, W13, W2, ids, w, act, dout, S13, S2)
        arr[idx] = old - h
        lm = _loss(x, W13, W2, ids, w, act, dout, S13, S2)
        arr[idx] = old
        return (lp - lm) / (2 * h)

    rng = np.random.default_rng(11)
    checks = [(x, g["dx"]), (W13, g["dw13"]), (W2, g["dw2"])]
    if shared:
        checks += [(S13, g["dw13_shared"]), (S2, g["dw2_shared"])]
    for arr, grad in checks:
        for _ in range(12):
            idx = tuple(int(rng.integers(0, n)) for n in arr.shape)
            assert fd(arr, idx) == pytest.approx(grad[idx], rel=1e-6, abs=1e-7), idx


def _torch_forward(x, W13, W2, ids, w, act, S13=None, S2=None):
    """The layer from its definition, in torch fp64: per token, the weighted
    sum of its k experts' MLPs (plus the shared expert's)."""
    T = x.shape[0]
    outs = []
    for t in range(T):
        acc = torch.zeros(x.shape[1], dtype=torch.float64)
        for j in range(ids.shape[1]):
            e = int(ids[t, j])
            a = W13[e] @ x[t]
            if act == oracle.ACT_SWIGLU:
                F = W13.shape[1] // 2
                hh = torch.nn.functional.silu(a[:F]) * a[F:]
            else:
                hh = torch.relu(a) ** 2
            acc = acc + w[t, j] * (W2[e] @ hh)
        if S13 is not None:
            a = S13[0] @ x[t]
            if act == oracle.ACT_SWIGLU:
                F = S13.shape[1] // 2
                hh = torch.nn.functional.silu(a[:F]) * a[F:]
            else:
                hh = torch.relu(a) ** 2
            acc = acc + S2[0] @ hh
        outs.append(acc)
    return torch.stack(outs)


@pytest.mark.parametrize("act", ACTS)
@pytest.mark.parametrize("shared", [False, True])
def test_matches_torch_autograd(act, shared):
    x, W13, W2, ids, w, dout, S13, S2 = _problem(4, act, T=7, d=8, F=6, E=4, k=3, shared=shared)
    g = oracle.backward_values(x, W13, W2, ids, w, act, dout, S13, S2)
    tx, t13, t2, tw = (torch.tensor(a, requires_grad=True) for a in (x, W13, W2, w))
    ts13 = torch.tensor(S13, requires_grad=True) if shared else None
    ts2 = torch.tensor(S2, requires_grad=True) if shared else None
    out = _torch_forward(tx, t13, t2, ids, tw, act, ts13, ts2)
    (out * torch.tensor(dout)).sum().backward()
    np.testing.assert_allclose(g["dx"], tx.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(g["dw13"], t13.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(g["dw2"], t2.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(g["dtopk_weights"], tw.grad.numpy(), rtol=1e-10, atol=1e-12)
    if shared:
        np.testing.assert_allclose(g["dw13_shared"], ts13.grad.numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(g["dw2_shared"], ts2.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_unrouted_expert_has_zero_gradient_and_bits_wrapper_agrees():
    from grouped_gemm_gating_b200 import workloads as W
    x, W13, W2, ids, w, dout, _, _ = _problem(5, oracle.ACT_SWIGLU, E=4, k=1)
    ids[:] = np.where(ids == 3, 0, ids)          # nobody routes to expert 3
    bits = lambda a: W.f32_to_bf16_bits(a.astype(np.float32))  # noqa: E731
    xb, w13b, w2b, db = bits(x), bits(W13), bits(W2), bits(dout)
    g = oracle.backward(xb, w13b, w2b, ids, w, oracle.ACT_SWIGLU, db)
    assert not g["dw13"][3].any() and not g["dw2"][3].any()
    gv = oracle.backward_values(oracle.bf16_to_f64(xb), oracle.bf16_to_f64(w13b), oracle.bf16_to_f64(w2b), ids, w,
                                oracle.ACT_SWIGLU, oracle.bf16_to_f64(db))
    for key in ("dx", "dw13", "dw2", "dtopk_weights"):
        assert np.array_equal(g[key], gv[key])


def test_silu_grad_against_central_difference():
    z = np.linspace(-8, 8, 33)
    h = 1e-6
    num = (oracle.silu(z + h) - oracle.silu(z - h)) / (2 * h)
    np.testing.assert_allclose(oracle.silu_grad(z), num, rtol=1e-7, atol=1e-9)
