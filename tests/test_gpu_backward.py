"""Parity of the backward pass (moe_backward, through the C ABI) with the
fp64 oracle's chain rule.

Each gradient -- dx [T, d], dW13 [E, n1, d], dW2 [E, d, F] (and the shared
expert's), dL/d topk_weights [T, k] -- is compared element by element over
the whole tensor on reduced shapes that span several tiles in every
dimension with ragged edges, and on sampled tokens and experts at the zipf
training-forward prefill size.  Tolerance: the forward's (max |diff| within
2e-2 * rms(oracle) beyond the bf16 output's half ulp, relative L2 within
5e-3) plus, element-wise, 2^-8 of the sum of |terms| of the GEMM whose
operand (da, or w*h) the kernels round to bf16 (moe_testlib.compare_grad);
dL/d topk_weights is fp32 and compared without either allowance.
"""
import numpy as np
import pytest
import torch

import oracle
from grouped_gemm_gating_b200 import moe as M
from grouped_gemm_gating_b200 import workloads as W
from moe_testlib import DeviceLayer, bf16_dev, compare_grad, oracle_route

pytestmark = pytest.mark.gpu

CFG = W.CONFIGS
SMALL = {
    "bwd_swiglu": CFG["zipf"].with_(name="bwd_swiglu", T=300, d=256, F=192, E=8, k=2, seed=2201,
                                    logits_kind="normal"),
    "bwd_relu2": CFG["relu2"].with_(name="bwd_relu2", T=333, d=320, F=448, E=5, k=2, block_m=128, seed=2202),
    "bwd_shared": CFG["dsv3"].with_(name="bwd_shared", T=200, d=256, F=256, E=6, k=2, n_group=3, topk_group=2,
                                    seed=2203),
    "bwd_zipf_small": CFG["zipf"].with_(name="bwd_zipf_small", T=1000, d=256, F=192, E=32, k=4, seed=2204),
    "bwd_one_hot": CFG["tiny"].with_(name="bwd_one_hot", T=700, d=128, F=128, E=4, k=1, block_m=128, seed=2205,
                                     logits_kind="decode_hot"),
}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    M.load_library()


def _host(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _run(cfg, dout_bits):
    inp = W.make_inputs(cfg)
    lay = DeviceLayer(inp)
    lay.run()
    g = M.MoEGradBuffers(cfg.T, cfg.d, cfg.F, cfg.E, cfg.k, cfg.act, cfg.n_shared)
    g.backward(lay.buf, lay.x, lay.w13, lay.w2, bf16_dev(dout_bits), lay.w13s, lay.w2s)
    torch.cuda.synchronize()
    assert lay.status() == 0, M.status_name(lay.status())
    return inp, lay, g


def _abs_terms(inp, ids, w, dout_bits):
    """Per element, the sum of |terms| of each gradient GEMM whose rounded
    operand is da (dx, dW13) or w*h (dW2), from the oracle's da and h."""
    c = inp.cfg
    x = oracle.bf16_to_f64(inp.x)
    go = oracle.bf16_to_f64(dout_bits)
    w = np.asarray(w, dtype=np.float64)
    dx = np.zeros((c.T, c.d))
    d13 = {}
    d2 = {}
    for e in range(c.E):
        t_idx, j_idx = np.nonzero(ids == e)
        if t_idx.size == 0:
            continue
        W13 = oracle.bf16_to_f64(inp.w13[e])
        dy = w[t_idx, j_idx][:, None] * go[t_idx]
        da, h = oracle.expert_backward_hidden(x[t_idx], W13, oracle.bf16_to_f64(inp.w2[e]), dy, c.act)
        np.add.at(dx, t_idx, np.abs(da) @ np.abs(W13))
        d13[e] = np.abs(da).T @ np.abs(x[t_idx])
        d2[e] = np.abs(dy).T @ np.abs(h)
    if c.n_shared:
        W13 = oracle.bf16_to_f64(inp.w13_shared[0])
        da, h = oracle.expert_backward_hidden(x, W13, oracle.bf16_to_f64(inp.w2_shared[0]), go, c.act)
        dx += np.abs(da) @ np.abs(W13)
        d13["shared"] = np.abs(da).T @ np.abs(x)
        d2["shared"] = np.abs(go).T @ np.abs(h)
    return dx, d13, d2


def _compare_fp32(got, ref, label):
    diff = got.astype(np.float64) - ref
    rms = float(np.sqrt((ref ** 2).mean()))
    assert np.isfinite(got).all(), label
    assert float(np.abs(diff).max()) <= 2e-2 * rms, f"{label}: max|diff| {np.abs(diff).max() / rms:.3e} rms"
    assert float(np.linalg.norm(diff) / np.linalg.norm(ref)) <= 5e-3, label


@pytest.mark.parametrize("name", list(SMALL))
def test_backward_small_full_tensors(name):
    cfg = SMALL[name]
    dout = W.grad_output(cfg.T, cfg.d, seed=cfg.seed + 50)
    inp, lay, g = _run(cfg, dout)
    ids, w = oracle_route(inp)
    ref = oracle.backward(inp.x, inp.w13, inp.w2, ids, w, cfg.act, dout, inp.w13_shared, inp.w2_shared)
    adx, a13, a2 = _abs_terms(inp, ids, w, dout)
    compare_grad(_host(g.dx), ref["dx"], adx, f"{name} dx")
    hit = np.unique(ids)
    for e in range(cfg.E):
        if e in hit:
            compare_grad(_host(g.dw13[e]), ref["dw13"][e], a13[e], f"{name} dw13[{e}]")
            compare_grad(_host(g.dw2[e]), ref["dw2"][e], a2[e], f"{name} dw2[{e}]")
        else:  # no token routed to e: exactly zero
            assert not _host(g.dw13[e]).any() and not _host(g.dw2[e]).any(), f"{name}: expert {e} not zero"
    if cfg.n_shared:
        compare_grad(_host(g.dw13_shared[0]), ref["dw13_shared"][0], a13["shared"], f"{name} dw13_shared")
        compare_grad(_host(g.dw2_shared[0]), ref["dw2_shared"][0], a2["shared"], f"{name} dw2_shared")
    _compare_fp32(g.dtopk.cpu().numpy(), ref["dtopk_weights"], f"{name} dtopk")


def test_backward_zipf_full_size_sampled():
    """The zipf prefill (T=16384, d=2048, d_ff=768, E=128, k=8): dx and
    dL/dw on 64 seeded tokens (each from its own k rows), dW13 / dW2 of the
    four smallest hit experts and one mid-sized one over all their rows, and
    zero gradients for the experts no token reached."""
    cfg = CFG["zipf"]
    dout = W.grad_output(cfg.T, cfg.d, seed=cfg.seed + 50)
    inp, lay, g = _run(cfg, dout)
    ids = lay.buf.topk_ids.cpu().numpy()
    w = lay.buf.topk_weights.cpu().numpy().astype(np.float64)
    x = oracle.bf16_to_f64(inp.x)
    go = oracle.bf16_to_f64(dout)
    rng = np.random.default_rng(7)
    toks = np.sort(rng.choice(cfg.T, size=64, replace=False))
    dx_ref = np.zeros((toks.size, cfg.d))
    dx_abs = np.zeros((toks.size, cfg.d))
    dw_ref = np.zeros((toks.size, cfg.k))
    for i, t in enumerate(toks):
        for j in range(cfg.k):
            e = ids[t, j]
            W13 = oracle.bf16_to_f64(inp.w13[e])
            W2 = oracle.bf16_to_f64(inp.w2[e])
            gx, _, _, y = oracle.expert_backward_values(x[t:t + 1], W13, W2, w[t, j] * go[t:t + 1], cfg.act)
            da, _ = oracle.expert_backward_hidden(x[t:t + 1], W13, W2, w[t, j] * go[t:t + 1], cfg.act)
            dx_ref[i] += gx[0]
            dx_abs[i] += (np.abs(da) @ np.abs(W13))[0]
            dw_ref[i, j] = float(go[t] @ y[0])
    compare_grad(_host(g.dx)[toks], dx_ref, dx_abs, "zipf dx (sampled tokens)")
    _compare_fp32(g.dtopk.cpu().numpy()[toks], dw_ref, "zipf dtopk (sampled tokens)")
    counts = np.bincount(ids.ravel(), minlength=cfg.E)
    hit = np.nonzero(counts)[0]
    by_size = hit[np.argsort(counts[hit], kind="stable")]
    for e in list(by_size[:4]) + [by_size[len(by_size) // 2]]:
        t_idx, j_idx = np.nonzero(ids == e)
        W13 = oracle.bf16_to_f64(inp.w13[e])
        W2 = oracle.bf16_to_f64(inp.w2[e])
        dy = w[t_idx, j_idx][:, None] * go[t_idx]
        _, gw13, gw2, _ = oracle.expert_backward_values(x[t_idx], W13, W2, dy, cfg.act)
        da, h = oracle.expert_backward_hidden(x[t_idx], W13, W2, dy, cfg.act)
        compare_grad(_host(g.dw13[e]), gw13, np.abs(da).T @ np.abs(x[t_idx]), f"zipf dw13[{e}] ({t_idx.size} rows)")
        compare_grad(_host(g.dw2[e]), gw2, np.abs(dy).T @ np.abs(h), f"zipf dw2[{e}] ({t_idx.size} rows)")
    for e in np.nonzero(counts == 0)[0]:
        assert not _host(g.dw13[e]).any() and not _host(g.dw2[e]).any()


def test_backward_is_repeatable_on_one_workspace():
    """Two calls on the same buffers: the weight gradients are one fp32 sum
    each in a fixed order (bit-identical); dx's k terms are added with
    atomics (within one bf16 ulp plus 1e-4 rms)."""
    from moe_testlib import assert_within_ulp
    cfg = SMALL["bwd_zipf_small"]
    dout = bf16_dev(W.grad_output(cfg.T, cfg.d, seed=cfg.seed + 50))
    inp = W.make_inputs(cfg)
    lay = DeviceLayer(inp)
    lay.run()
    g = M.MoEGradBuffers(cfg.T, cfg.d, cfg.F, cfg.E, cfg.k, cfg.act, cfg.n_shared)
    g.backward(lay.buf, lay.x, lay.w13, lay.w2, dout)
    first = [_host(t).copy() for t in (g.dx, g.dw13, g.dw2)]
    g.backward(lay.buf, lay.x, lay.w13, lay.w2, dout)
    torch.cuda.synchronize()
    assert lay.status() == 0
    assert_within_ulp(_host(g.dx), first[0], 1, "dx")
    assert np.array_equal(_host(g.dw13), first[1]) and np.array_equal(_host(g.dw2), first[2])
