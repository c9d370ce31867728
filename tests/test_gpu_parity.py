"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle.

Routing ids, align outputs: bit-exact.  Routing weights: within
WEIGHT_TOL * max(1, |w|).  Layer output: max |diff| <= 2e-2 * rms(oracle)
and relative L2 <= 5e-3.  Small cases are compared element by element over
the whole output; the full-size workloads on a seeded sample of tokens.
"""
import numpy as np
import pytest
import torch

import oracle
from grouped_gemm_gating_b200 import moe as M
from grouped_gemm_gating_b200 import workloads as W
from moe_testlib import (DeviceLayer, assert_within_ulp, compare_align, compare_out, compare_route,
                         oracle_route, route_kwargs)

pytestmark = pytest.mark.gpu

CFG = W.CONFIGS

# Reduced versions of every configuration: the oracle finishes them in
# seconds, yet they span several tiles in both dimensions and ragged tails.
SMALL = {
    "tiny": CFG["tiny"],
    "decode": CFG["decode"],
    "decode_d512": CFG["decode"].with_(name="decode_d512", d=512, F=384, seed=2002),
    "relu2_small": CFG["relu2"].with_(name="relu2_small", T=64, E=16, seed=2004),
    "dsv3_small": CFG["dsv3"].with_(name="dsv3_small", T=300, d=512, F=384, seed=2003),
    "zipf_small": CFG["zipf"].with_(name="zipf_small", T=1000, d=256, F=192, E=32, seed=2005,
                                    logits_kind="normal"),
    "swap_bm32": CFG["tiny"].with_(name="swap_bm32", T=200, d=256, F=320, E=8, k=3, block_m=32, seed=2006,
                                   logits_kind="normal"),
    "swap_bm64_relu2": CFG["relu2"].with_(name="swap_bm64_relu2", T=150, d=192, F=192, E=6, k=2, block_m=64,
                                          seed=2007),
    "tokm_relu2": CFG["relu2"].with_(name="tokm_relu2", T=333, d=320, F=448, E=5, k=2, block_m=128,
                                     seed=2008),
    "one_expert_hot": CFG["tiny"].with_(name="one_expert_hot", T=700, d=128, F=128, E=4, k=1, block_m=128,
                                        seed=2009, logits_kind="decode_hot"),
    # token-major GEMMs on CTA pairs (d, d_ff >= 1024), odd and even block
    # runs per expert, a shared expert, and the relu^2 variant
    "pair_dsv3": CFG["dsv3"].with_(name="pair_dsv3", T=600, d=1024, F=1024, seed=2012),
    "pair_relu2": CFG["relu2"].with_(name="pair_relu2", T=400, d=1024, F=1088, E=6, k=2, block_m=128,
                                     seed=2013),
    # fused expert kernel (block_m <= 64) with a shared expert
    "shared_bm16_fused_combine": CFG["dsv3"].with_(name="shared_bm16_fused_combine", T=40, d=256, F=192,
                                                   block_m=16, seed=2010),
    "shared_bm32_sep_combine": CFG["dsv3"].with_(name="shared_bm32_sep_combine", T=100, d=320, F=128,
                                                 block_m=32, seed=2011),
    # the header's limits: E = 256 experts, top_k = 16, T*k = 256 slots (the
    # largest one-launch moe_layer), grouped routing, a last h slice past d_ff
    "limits_e256_k16": CFG["decode"].with_(name="limits_e256_k16", T=16, d=256, F=192, E=256, k=16, n_group=8,
                                           topk_group=4, seed=2014, logits_kind="normal"),
    # SwiGLU in the fused kernel with 64-token blocks and a half-empty last slice
    "swap_bm64_swiglu": CFG["tiny"].with_(name="swap_bm64_swiglu", T=150, d=192, F=320, E=6, k=2, block_m=64,
                                          seed=2015, logits_kind="normal"),
}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    M.load_library()


def _full_check(cfg):
    inp = W.make_inputs(cfg)
    lay = DeviceLayer(inp)
    out = lay.run()
    torch.cuda.synchronize()
    assert lay.status() == 0, M.status_name(lay.status())
    ids, w = oracle_route(inp)
    compare_route(lay.buf.topk_ids.cpu().numpy(), lay.buf.topk_weights.cpu().numpy(), ids, w, cfg.name)
    compare_align(lay.buf, oracle.align(ids, cfg.E, cfg.block_m), cfg.name)
    ref = oracle.forward(inp.x, inp.w13, inp.w2, ids, w, cfg.act, inp.w13_shared, inp.w2_shared)
    return compare_out(M_bits(out), ref, cfg.name)


def M_bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("name", list(SMALL))
def test_layer_small_full_output(name):
    _full_check(SMALL[name])


def test_hidden_activation_matches_oracle():
    """h rows (first GEMM + activation) checked on their own."""
    cfg = SMALL["dsv3_small"]
    inp = W.make_inputs(cfg)
    lay = DeviceLayer(inp)
    lay.run()
    torch.cuda.synchronize()
    ids, _ = oracle_route(inp)
    st = lay.buf.sorted_token_ids.cpu().numpy()
    ex = lay.buf.expert_ids.cpu().numpy()
    ntpp = int(lay.buf.ntpp.item())
    h = lay.h_rows()
    x = oracle.bf16_to_f64(inp.x)
    S = cfg.T * cfg.k
    rng = np.random.default_rng(0)
    for p in rng.choice(ntpp, size=64, replace=False):
        s = st[p]
        if s >= S:
            assert np.all(h[p] == 0.0), "padding rows of h must be zero"
            continue
        ref = oracle.expert_hidden(x[s // cfg.k][None, :], inp.w13[ex[p // cfg.block_m]], cfg.act)[0]
        err = np.abs(h[p] - ref).max()
        assert err <= 1e-2 * max(np.abs(ref).max(), 1e-3), (p, err)
    # shared-expert rows follow the routed rows
    for t in (0, cfg.T - 1):
        ref = oracle.expert_hidden(x[t][None, :], inp.w13_shared[0], cfg.act)[0]
        assert np.abs(h[ntpp + t] - ref).max() <= 1e-2 * np.abs(ref).max()


# ------------------------------------------------------------ routing -----

@pytest.mark.parametrize("name", list(CFG))
def test_route_parity_configs(name):
    cfg = CFG[name]
    rng_inp = W.make_inputs(cfg.with_(d=64, F=64, E=cfg.E)) if name != "tiny" else W.make_inputs(cfg)
    lg = rng_inp.logits
    dev = torch.from_numpy(lg).cuda()
    ids = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moe_route(dev, cfg.k, ids, w, dev_status=st, **route_kwargs(cfg))
    assert M.moe_read_status(st) == 0
    ref = oracle.route(lg, cfg.k, cfg.n_group, cfg.topk_group, cfg.group_score, bool(cfg.renormalize),
                       cfg.routed_scaling)
    compare_route(ids.cpu().numpy(), w.cpu().numpy(), *ref, name)


@pytest.mark.parametrize("E,k,n_group,topk_group,score,renorm,scale", [
    (8, 2, 1, 1, 0, 1, 1.0),
    (16, 4, 4, 2, 0, 1, 2.5),
    (16, 4, 4, 2, 1, 1, 1.0),
    (18, 4, 6, 4, 1, 0, 1.0),
    (64, 6, 8, 3, 0, 0, 1.0),
    (128, 8, 1, 1, 0, 0, 2.5),
    (256, 16, 8, 4, 1, 1, 1.0),
    (256, 8, 256, 8, 0, 1, 1.0),
    (5, 5, 1, 1, 0, 1, 1.0),
    (1, 1, 1, 1, 0, 1, 1.0),
])
@pytest.mark.parametrize("ties", [False, True])
def test_route_parity_variants(E, k, n_group, topk_group, score, renorm, scale, ties):
    T = 333
    lg = W.tie_logits(T, E, seed=E + k, levels=3) if ties else \
        np.random.default_rng(E * 7 + k).standard_normal((T, E)).astype(np.float32)
    dev = torch.from_numpy(lg).cuda()
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    M.moe_route(dev, k, ids, w, n_group, topk_group, score, bool(renorm), scale)
    ref = oracle.route(lg, k, n_group, topk_group, score, bool(renorm), scale)
    compare_route(ids.cpu().numpy(), w.cpu().numpy(), *ref, f"E{E}k{k}g{n_group}")


def test_route_nonfinite_sets_status():
    lg = np.zeros((4, 8), np.float32)
    lg[2, 3] = np.nan
    ids = torch.empty((4, 2), dtype=torch.int32, device="cuda")
    w = torch.empty((4, 2), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moe_route(torch.from_numpy(lg).cuda(), 2, ids, w, dev_status=st)
    assert M.moe_read_status(st) == 5


# ------------------------------------------------------------- align ------

def _align_gpu(ids_np, E, bm):
    T, k = ids_np.shape
    buf = M.MoEBuffers(T, 64, 64, E, k, bm)
    buf.topk_ids.copy_(torch.from_numpy(ids_np))
    buf.align()
    torch.cuda.synchronize()
    assert M.moe_read_status(buf.status) == 0
    return buf


@pytest.mark.parametrize("bm", [16, 32, 64, 128])
@pytest.mark.parametrize("T,E,k,skew", [
    (1, 8, 1, 0.0), (3, 128, 8, 0.0), (256, 128, 6, 0.0), (1024, 8, 8, 3.0), (1023, 256, 8, 0.0),
    (1025, 256, 8, 50.0), (2048, 128, 8, 0.0), (4096, 18, 4, 0.0), (16384, 128, 8, 5.0),
    (5000, 32, 3, 0.0),
])
def test_align_parity(bm, T, E, k, skew):
    ids = W.random_topk_ids(T, E, k, seed=T + E + bm, skew=skew)
    buf = _align_gpu(ids, E, bm)
    compare_align(buf, oracle.align(ids, E, bm), f"T{T}E{E}k{k}bm{bm}")


def test_align_all_slots_one_expert_and_empty():
    T, E, k, bm = 9000, 64, 1, 128          # multi-chunk path, one expert owns all slots
    ids = np.full((T, k), 17, np.int32)
    compare_align(_align_gpu(ids, E, bm), oracle.align(ids, E, bm), "one-expert")
    ids = np.zeros((0, 4), np.int32)
    buf = M.MoEBuffers(0, 64, 64, 16, 4, 16)
    buf.align()
    torch.cuda.synchronize()
    compare_align(buf, oracle.align(ids, 16, 16), "empty")


def test_align_bad_expert_id_sets_status():
    ids = np.array([[0, 1], [2, 99]], np.int32)
    buf = M.MoEBuffers(2, 64, 64, 8, 2, 16)
    buf.topk_ids.copy_(torch.from_numpy(ids))
    buf.align()
    assert M.moe_read_status(buf.status) == 7


# -------------------------------------------------------- full size -------

@pytest.mark.slow
@pytest.mark.parametrize("name", ["decode", "relu2", "dsv3", "zipf"])
def test_layer_full_size_sampled(name):
    """Full-size workload in the benchmark's launch configuration; the oracle
    checks routing and align in full and the output on sampled tokens."""
    cfg = CFG[name]
    inp = W.make_inputs(cfg)
    lay = DeviceLayer(inp)
    out = lay.run()
    torch.cuda.synchronize()
    assert lay.status() == 0, M.status_name(lay.status())
    ids, w = oracle_route(inp)
    compare_route(lay.buf.topk_ids.cpu().numpy(), lay.buf.topk_weights.cpu().numpy(), ids, w, name)
    compare_align(lay.buf, oracle.align(ids, cfg.E, cfg.block_m), name)
    n = min(cfg.T, 96)
    sample = np.sort(np.random.default_rng(cfg.seed).choice(cfg.T, size=n, replace=False))
    ref = oracle.forward(inp.x[sample], inp.w13, inp.w2, ids[sample], w[sample], cfg.act,
                         inp.w13_shared, inp.w2_shared)
    compare_out(M_bits(out)[sample], ref, name)
    if name == "zipf":
        counts = np.bincount(ids.reshape(-1), minlength=cfg.E)
        assert (counts == 0).sum() == 8


@pytest.mark.slow
def test_layer_beyond_wide_gemm_block_limit_sampled():
    """More than 8192 blocks of 128 rows (T * k over a million slots): the
    gate/up GEMM runs on one-block tiles instead of two-block units."""
    cfg = CFG["tiny"].with_(name="many_blocks", T=131072, d=128, F=128, E=8, k=8, block_m=128, seed=2016,
                            logits_kind="normal")
    inp = W.make_inputs(cfg)
    lay = DeviceLayer(inp)
    out = lay.run()
    torch.cuda.synchronize()
    assert lay.status() == 0, M.status_name(lay.status())
    ids, w = oracle_route(inp)
    assert M.moe_max_padded(cfg.T, cfg.k, cfg.E, cfg.block_m) // cfg.block_m > 8192
    compare_align(lay.buf, oracle.align(ids, cfg.E, cfg.block_m), cfg.name)
    sample = np.sort(np.random.default_rng(cfg.seed).choice(cfg.T, size=64, replace=False))
    ref = oracle.forward(inp.x[sample], inp.w13, inp.w2, ids[sample], w[sample], cfg.act)
    compare_out(M_bits(out)[sample], ref, cfg.name)


def test_repeated_calls_agree_up_to_sum_order():
    """Both paths add partial sums with fp32 atomics in a timing-dependent
    order: repeated calls agree up to that reordering (a bf16 ulp of the
    result, 1e-4 rms where terms cancel); routing / align outputs are
    bit-identical."""
    for name in ("zipf_small", "decode_d512"):
        lay = DeviceLayer(W.make_inputs(SMALL[name]))
        a = M_bits(lay.run()).copy()
        ids = lay.buf.sorted_token_ids.clone()
        for _ in range(3):
            assert_within_ulp(M_bits(lay.run()), a, 1, name)
            assert torch.equal(lay.buf.sorted_token_ids, ids)


def test_forward_zero_tokens_is_noop():
    buf = M.MoEBuffers(0, 128, 128, 8, 2, 16)
    x = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    w13 = torch.zeros((8, 256, 128), dtype=torch.bfloat16, device="cuda")
    w2 = torch.zeros((8, 128, 128), dtype=torch.bfloat16, device="cuda")
    buf.align()
    buf.forward(x, w13, w2)
    torch.cuda.synchronize()


def test_cuda_graph_replay_matches_eager():
    """The three calls capture into a CUDA graph (PDL edges included); a
    replay on new inputs matches the eager result bit for bit."""
    cfg = SMALL["decode_d512"]
    inp = W.make_inputs(cfg)
    lay = DeviceLayer(inp)
    lay.run()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        lay.run()
    inp2 = W.make_inputs(cfg.with_(seed=cfg.seed + 1))
    lay.x.copy_(torch.from_numpy(inp2.x.view(np.int16)).cuda().view(torch.bfloat16))
    lay.logits.copy_(torch.from_numpy(inp2.logits).cuda())
    g.replay()
    torch.cuda.synchronize()
    replayed = M_bits(lay.buf.out).copy()
    eager = M_bits(lay.run()).copy()
    # partial sums are added with fp32 atomics: equal up to their reordering
    assert_within_ulp(replayed, eager, 1)
    ids, w = oracle_route(inp2)
    ref = oracle.forward(inp2.x, inp.w13, inp.w2, ids, w, cfg.act)
    compare_out(replayed, ref, "graph replay")


def test_profile_events_cover_every_kernel():
    cfg = SMALL["zipf_small"]
    lay = DeviceLayer(W.make_inputs(cfg))
    lay.run()
    M.moe_profile_enable(True)
    lay.run()
    M.moe_profile_enable(False)
    st = M.moe_profile_collect()
    assert st["route"][1] == 1 and st["gate_up_gemm"][1] == 1 and st["down_gemm"][1] == 1
    assert st["combine"][1] == 1 and st["align"][1] == 1
    assert all(ms > 0.0 for ms, n in st.values() if n)
    # the small-batch path: one fused route+align kernel, one fused expert kernel
    lay = DeviceLayer(W.make_inputs(SMALL["decode"]))
    lay.buf.route_align(lay.logits)
    lay.buf.forward(lay.x, lay.w13, lay.w2)
    M.moe_profile_enable(True)
    lay.buf.route_align(lay.logits)
    lay.buf.forward(lay.x, lay.w13, lay.w2)
    M.moe_profile_enable(False)
    st = M.moe_profile_collect()
    assert st["route_align"][1] == 1 and st["fused_expert"][1] == 1
    assert st["combine"][1] == 0 and st["gate_up_gemm"][1] == 0


@pytest.mark.parametrize("name,T", [("tiny", None), ("decode", None), ("relu2_small", None), ("dsv3_small", 16),
                                    ("dsv3_small", 300), ("swap_bm32", 64), ("zipf_small", None)])
def test_route_align_matches_separate_calls(name, T):
    cfg = SMALL[name] if T is None else SMALL[name].with_(T=T)
    inp = W.make_inputs(cfg)
    a = DeviceLayer(inp)
    b = DeviceLayer(inp)
    a.buf.route(a.logits, **route_kwargs(cfg))
    a.buf.align()
    b.buf.route_align(b.logits, **route_kwargs(cfg))
    torch.cuda.synchronize()
    assert b.status() == 0
    S = cfg.T * cfg.k
    for attr in ("topk_ids", "topk_weights", "sorted_token_ids", "expert_ids", "ntpp"):
        x, y = getattr(a.buf, attr), getattr(b.buf, attr)
        assert torch.equal(x.view(torch.int32), y.view(torch.int32)), attr
    assert torch.equal(a.buf.inv_pos[:S], b.buf.inv_pos[:S])
    ids, w = oracle_route(inp)
    compare_route(b.buf.topk_ids.cpu().numpy(), b.buf.topk_weights.cpu().numpy(), ids, w, name)


@pytest.mark.parametrize("name,one_launch", [("decode", True), ("tiny", True), ("shared_bm16_fused_combine", True),
                                             ("decode_d512", True), ("limits_e256_k16", True), ("relu2_small", False),
                                             ("dsv3_small", False), ("swap_bm32", False)])
def test_layer_entry_matches_separate_calls(name, one_launch):
    """moe_layer writes the same routing / align outputs as moe_route_align
    (bit for bit) and the same output as moe_forward (up to the reordering
    of fp32 sums); small decode batches take one launch."""
    cfg = SMALL[name]
    inp = W.make_inputs(cfg)
    a = DeviceLayer(inp)
    b = DeviceLayer(inp)
    ref_out = M_bits(a.run(fused_route_align=True)).copy()
    rk = route_kwargs(cfg)
    b.buf.layer(b.logits, b.x, b.w13, b.w2, b.w13s, b.w2s, **rk)
    torch.cuda.synchronize()
    if one_launch:
        assert M.moe_last_launch_count() == 1
    assert b.status() == 0, M.status_name(b.status())
    S = cfg.T * cfg.k
    for attr in ("topk_ids", "topk_weights", "sorted_token_ids", "expert_ids", "ntpp"):
        x, y = getattr(a.buf, attr), getattr(b.buf, attr)
        assert torch.equal(x.view(torch.int32), y.view(torch.int32)), attr
    assert torch.equal(a.buf.inv_pos[:S], b.buf.inv_pos[:S])
    got = M_bits(b.buf.out).copy()
    assert_within_ulp(got, ref_out, 1, name)
    ids, w = oracle_route(inp)
    ref = oracle.forward(inp.x, inp.w13, inp.w2, ids, w, cfg.act, inp.w13_shared, inp.w2_shared)
    compare_out(got, ref, name + " (moe_layer)")


def test_layer_entry_graph_replay():
    """The one-launch layer captures into a CUDA graph and replays on new
    logits and activations."""
    cfg = SMALL["decode_d512"]
    inp = W.make_inputs(cfg)
    lay = DeviceLayer(inp)
    lay.buf.layer(lay.logits, lay.x, lay.w13, lay.w2)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        lay.buf.layer(lay.logits, lay.x, lay.w13, lay.w2)
    inp2 = W.make_inputs(cfg.with_(seed=cfg.seed + 7))
    lay.x.copy_(torch.from_numpy(inp2.x.view(np.int16)).cuda().view(torch.bfloat16))
    lay.logits.copy_(torch.from_numpy(inp2.logits).cuda())
    g.replay()
    torch.cuda.synchronize()
    assert lay.status() == 0
    ids, w = oracle_route(inp2)
    compare_route(lay.buf.topk_ids.cpu().numpy(), lay.buf.topk_weights.cpu().numpy(), ids, w, "layer replay")
    compare_align(lay.buf, oracle.align(ids, cfg.E, cfg.block_m), "layer replay")
    ref = oracle.forward(inp2.x, inp.w13, inp.w2, ids, w, cfg.act)
    compare_out(M_bits(lay.buf.out), ref, "layer replay")


def test_fused_counters_return_to_zero_and_workspace_is_shareable():
    """The fused kernel's grid counters are zero after every call (the third
    word is a release generation that only moves forward; the rest of the
    block stays zero), so one workspace serves calls of different shapes in
    turn."""
    cfg_a = SMALL["decode_d512"]
    cfg_b = SMALL["swap_bm32"]
    lay_a = DeviceLayer(W.make_inputs(cfg_a))
    lay_b = DeviceLayer(W.make_inputs(cfg_b))
    shared_ws = lay_a.buf.ws if lay_a.buf.ws.numel() >= lay_b.buf.ws.numel() else lay_b.buf.ws
    lay_a.buf.ws = shared_ws
    lay_b.buf.ws = shared_ws
    ref_a = M_bits(lay_a.run()).copy()
    ref_b = M_bits(lay_b.run()).copy()
    for _ in range(2):
        assert_within_ulp(M_bits(lay_a.run()), ref_a, 1)
        torch.cuda.synchronize()
        base = (shared_ws.data_ptr() + 255) // 256 * 256 - shared_ws.data_ptr()
        words = shared_ws[base: base + 65536].view(torch.int32)
        assert int(words[:2].count_nonzero()) == 0 and int(words[3:].count_nonzero()) == 0
        assert_within_ulp(M_bits(lay_b.run()), ref_b, 1)
    assert lay_a.status() == 0 and lay_b.status() == 0
