"""GPU parity of moe_router (router projection + top-k gating) through the C ABI.

The logits are checked against the fp64 oracle within the error bound of
fp32 accumulation: the bf16 products are exact in fp32 and each of the d
additions rounds once, so |gpu - exact| <= d * 2^-24 * sum_i |x_i w_i|.
The gating is an integer decision taken on those fp32 logits, so the oracle
routes the GPU's own logits: ids bit for bit, weights within the routing
tolerance.  The same logits through moe_route give the same ids.
"""
import numpy as np
import pytest
import torch

import oracle
from grouped_gemm_gating_b200 import moe as M
from grouped_gemm_gating_b200 import workloads as W
from moe_testlib import compare_route

pytestmark = pytest.mark.gpu


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _run(T, d, E, k, n_group=1, topk_group=1, score=0, renorm=True, scale=1.0, seed=0, zero_rows=()):
    x, w = W.router_inputs(T, d, E, seed=seed, zero_rows=zero_rows)
    logits = torch.full((T, E), float("nan"), dtype=torch.float32, device="cuda")
    ids = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    wts = torch.full((T, k), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moe_router(_dev_bf16(x), _dev_bf16(w), k, logits, ids, wts, n_group, topk_group, score, renorm, scale, st)
    assert M.moe_read_status(st) == 0, M.status_name(M.moe_read_status(st))
    lg = logits.cpu().numpy()
    exact = oracle.router_logits(x, w)
    bound = d * 2.0 ** -24 * (np.abs(oracle.bf16_to_f64(x)) @ np.abs(oracle.bf16_to_f64(w)).T) + 1e-30
    err = np.abs(lg.astype(np.float64) - exact)
    assert (err <= bound).all(), f"logits beyond the fp32 accumulation bound at {np.argwhere(err > bound)[:5]}"
    ref_ids, ref_w = oracle.route(lg, k, n_group, topk_group, score, renorm, scale)
    compare_route(ids.cpu().numpy(), wts.cpu().numpy(), ref_ids, ref_w, f"router T{T} d{d} E{E} k{k}")
    # the routing kernel on the same logits picks the same experts
    ids2 = torch.empty_like(ids)
    w2 = torch.empty_like(wts)
    M.moe_route(logits, k, ids2, w2, n_group, topk_group, score, renorm, scale)
    assert torch.equal(ids2, ids)
    return lg


@pytest.mark.parametrize("T,d,E,k", [
    (32, 128, 8, 2),      # the tiny layer's router shape (CUDA-core product, two token chunks)
    (3, 2048, 128, 8),    # decode batch
    (16, 2688, 128, 6),   # one full chunk of 16 tokens, d = 2688
    (300, 512, 18, 4),    # E not a multiple of 8, a ragged last chunk
    (130, 256, 256, 16),  # the limits: E = 256, k = 16
    (1, 64, 1, 1),
    (1024, 256, 40, 3),   # the largest CUDA-core batch
    (1025, 256, 40, 3),   # the smallest tensor-core batch, a ragged last tile
    (5000, 512, 18, 4),   # tensor cores, E not a multiple of 16
])
def test_router_parity(T, d, E, k):
    _run(T, d, E, k, seed=T * 7 + E)


@pytest.mark.parametrize("T", [200, 4200])
def test_router_full_softmax_and_scaling(T):
    _run(T, 256, 64, 6, renorm=False, scale=2.5, seed=5)


@pytest.mark.parametrize("T", [257, 4500])
def test_router_grouped_runs_the_routing_kernel_on_its_logits(T):
    _run(T, 384, 18, 4, n_group=6, topk_group=4, score=1, seed=6)


@pytest.mark.parametrize("T", [40, 4100])
def test_router_zero_token_ties_to_lowest_ids(T):
    # a zero token scores every expert 0: the gating keeps experts 0..k-1
    lg = _run(T, 128, 32, 5, seed=7, zero_rows=(0, 17, 39))
    assert (lg[[0, 17, 39]] == 0).all()


def test_router_zero_tokens_is_noop():
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((8, 64), dtype=torch.bfloat16, device="cuda")
    lg = torch.zeros((0, 8), dtype=torch.float32, device="cuda")
    ids = torch.zeros((0, 2), dtype=torch.int32, device="cuda")
    wts = torch.zeros((0, 2), dtype=torch.float32, device="cuda")
    M.moe_router(x, w, 2, lg, ids, wts)
    torch.cuda.synchronize()
