"""Parity of the fp8-weight layer (moe_layer_fp8 / moe_forward_fp8, through
the C ABI) with the fp64 oracle on the dequantised weights.

The weights are quantised once on the host (workloads.quantize_mxfp8: e4m3
values, one power-of-two scale per 32 K values of a row); the oracle decodes
the same bytes (oracle.dequant_mxfp8) and runs its forward on them.  The
kernel's expansion to bf16 is exact, so the tolerance is the bf16 layer's,
and the fp8 layer must agree with the bf16 layer run on the dequantised
weights up to the fp32 reordering of the scatter-reduce.
"""
import numpy as np
import pytest
import torch

import oracle
from grouped_gemm_gating_b200 import moe as M
from grouped_gemm_gating_b200 import workloads as W
from moe_testlib import assert_within_ulp, bf16_dev, compare_align, compare_out, compare_route, oracle_route, \
    route_kwargs

pytestmark = pytest.mark.gpu

CFG = W.CONFIGS
CASES = {
    "decode": CFG["decode"],
    "relu2": CFG["relu2"],
    "tiny": CFG["tiny"],
    "fp8_bm32": CFG["tiny"].with_(name="fp8_bm32", T=200, d=256, F=320, E=8, k=3, block_m=32, seed=2306,
                                  logits_kind="normal"),
    "fp8_bm64_relu2": CFG["relu2"].with_(name="fp8_bm64_relu2", T=150, d=192, F=192, E=6, k=2, block_m=64,
                                         seed=2307),
    "fp8_shared_bm16": CFG["dsv3"].with_(name="fp8_shared_bm16", T=40, d=256, F=192, block_m=16, seed=2310),
    "fp8_limits_e256_k16": CFG["decode"].with_(name="fp8_limits_e256_k16", T=16, d=256, F=192, E=256, k=16,
                                               n_group=8, topk_group=4, seed=2314, logits_kind="normal"),
}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    M.load_library()


def _u8(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


# full-output comparison up to this many tokens; larger batches on a seeded sample
FULL_TOKENS = 64
SAMPLE_TOKENS = 24


def _setup(cfg):
    inp = W.make_inputs(cfg)
    q = W.fp8_weights(inp)
    wq = M.Fp8Experts(*[None if a is None else _u8(a) for a in q])
    return inp, wq, q


def _oracle_out(inp, q, ids, w, tokens):
    """The oracle's forward on the dequantised weights for the given tokens
    (only the experts they reach are dequantised)."""
    c = inp.cfg
    sub = ids[tokens]
    hit = np.unique(sub)
    W13 = np.zeros((c.E, c.n1, c.d))
    W2 = np.zeros((c.E, c.d, c.F))
    W13[hit] = oracle.dequant_mxfp8(q[0][hit], q[1][hit])
    W2[hit] = oracle.dequant_mxfp8(q[2][hit], q[3][hit])
    sh = (None, None) if q[4] is None else (oracle.dequant_mxfp8(q[4], q[5]), oracle.dequant_mxfp8(q[6], q[7]))
    return oracle.forward_values(oracle.bf16_to_f64(inp.x[tokens]), W13, W2, sub, w[tokens], c.act, *sh)


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("name", list(CASES))
def test_fp8_layer_matches_oracle_on_dequantised_weights(name):
    cfg = CASES[name]
    inp, wq, q = _setup(cfg)
    buf = M.MoEBuffers(cfg.T, cfg.d, cfg.F, cfg.E, cfg.k, cfg.block_m, cfg.act, cfg.n_shared)
    x = bf16_dev(inp.x)
    logits = torch.from_numpy(inp.logits).cuda()
    out = buf.layer_fp8(logits, x, wq, **route_kwargs(cfg))
    torch.cuda.synchronize()
    assert M.moe_read_status(buf.status) == 0, M.status_name(M.moe_read_status(buf.status))
    ids, w = oracle_route(inp)
    compare_route(buf.topk_ids.cpu().numpy(), buf.topk_weights.cpu().numpy(), ids, w, name)
    compare_align(buf, oracle.align(ids, cfg.E, cfg.block_m), name)
    tokens = np.arange(cfg.T) if cfg.T <= FULL_TOKENS else \
        np.sort(np.random.default_rng(cfg.seed).choice(cfg.T, size=SAMPLE_TOKENS, replace=False))
    compare_out(_bits(out)[tokens], _oracle_out(inp, q, ids, w, tokens), f"{name} (fp8)")
    # separate forward call on the same routing: the same result
    out2 = _bits(buf.forward_fp8(x, wq)).copy()
    torch.cuda.synchronize()
    assert M.moe_read_status(buf.status) == 0
    assert_within_ulp(out2, _bits(out), 1, f"{name} forward_fp8 vs layer_fp8")


@pytest.mark.parametrize("name", ["decode", "fp8_bm32"])
def test_fp8_equals_bf16_layer_on_dequantised_weights(name):
    """The expansion to bf16 is exact: the fp8 layer and the bf16 layer on
    bf16(dequantised weights) differ only by the scatter-reduce's order."""
    cfg = CASES[name]
    inp, wq, q = _setup(cfg)
    w13, w2 = oracle.dequant_mxfp8(q[0], q[1]), oracle.dequant_mxfp8(q[2], q[3])
    as_bf16 = lambda a: bf16_dev(W.f32_to_bf16_bits(a.astype(np.float32)))  # noqa: E731
    assert np.array_equal(W.bf16_bits_to_f32(W.f32_to_bf16_bits(w13.astype(np.float32))), w13)  # exact in bf16
    x = bf16_dev(inp.x)
    logits = torch.from_numpy(inp.logits).cuda()
    b8 = M.MoEBuffers(cfg.T, cfg.d, cfg.F, cfg.E, cfg.k, cfg.block_m, cfg.act, cfg.n_shared)
    b16 = M.MoEBuffers(cfg.T, cfg.d, cfg.F, cfg.E, cfg.k, cfg.block_m, cfg.act, cfg.n_shared)
    o8 = _bits(b8.layer_fp8(logits, x, wq, **route_kwargs(cfg))).copy()
    o16 = _bits(b16.layer(logits, x, as_bf16(w13), as_bf16(w2), **route_kwargs(cfg))).copy()
    torch.cuda.synchronize()
    assert M.moe_read_status(b8.status) == 0 and M.moe_read_status(b16.status) == 0
    assert_within_ulp(o8, o16, 1, f"{name}: fp8 vs bf16 of the dequantised weights")


def test_fp8_rejects_prefill_blocks():
    cfg = CFG["tiny"].with_(name="fp8_bm128", block_m=128)
    inp, wq, _ = _setup(cfg)
    buf = M.MoEBuffers(cfg.T, cfg.d, cfg.F, cfg.E, cfg.k, 128, cfg.act, 0)
    with pytest.raises(M.MoEError) as ei:
        M.moe_forward_fp8(bf16_dev(inp.x), wq, buf.topk_weights, buf.sorted_token_ids, buf.expert_ids, buf.ntpp,
                          buf.inv_pos, 128, cfg.act, buf.out, buf.ws)
    assert ei.value.code == 2   # MOE_ERR_UNSUPPORTED: fp8 weights run in the fused kernel (block_m <= 64)
