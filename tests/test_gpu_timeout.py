"""The bounded waits' error path, driven without faulting or hanging the GPU.

Every pipeline and grid wait inside the kernels gives up after a time limit,
records MOE_ERR_DEVICE_TIMEOUT, waits for its own TMA loads and MMAs still
in flight, frees its tensor memory and returns.  The test hook
moe_debug_timeouts lowers that limit and can make the fused expert kernel's
start barrier wait for one CTA more than the grid has (a count nothing
reaches).  Each test forces a timeout, checks the status and the workspace's
grid counters, then runs the same call again on the same workspace with the
default limit and checks the output against the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from grouped_gemm_gating_b200 import moe as M
from grouped_gemm_gating_b200 import workloads as W
from moe_testlib import DeviceLayer, compare_out, oracle_route, route_kwargs

pytestmark = pytest.mark.gpu

TIMEOUT = 6  # MOE_ERR_DEVICE_TIMEOUT


@pytest.fixture(autouse=True)
def _restore_limits():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    M.load_library()
    yield
    M.moe_debug_timeouts(0, 0)


def _counters(buf: M.MoEBuffers) -> np.ndarray:
    """The first words of the workspace's counter block (after rounding the
    workspace up to 256 bytes)."""
    off = (buf.ws.data_ptr() + 255) // 256 * 256 - buf.ws.data_ptr()
    return buf.ws[off: off + 16].view(torch.int32).cpu().numpy()


def _oracle_out(inp):
    c = inp.cfg
    ids, w = oracle_route(inp)
    return oracle.forward(inp.x, inp.w13, inp.w2, ids, w, c.act, inp.w13_shared, inp.w2_shared)


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _layer(lay: DeviceLayer):
    c = lay.cfg
    return lay.buf.layer(lay.logits, lay.x, lay.w13, lay.w2, lay.w13s, lay.w2s, **route_kwargs(c))


@pytest.mark.parametrize("use_layer", [True, False])
def test_fused_kernel_start_barrier_timeout_then_recovers(use_layer):
    """The decode shape: with use_layer the one-launch moe_layer (routing in
    the kernel, the last CTA converts the output); otherwise a 32-token-block
    forward whose CTAs are released by the generation word and convert their
    own slices."""
    cfg = W.CONFIGS["decode"] if use_layer else W.CONFIGS["tiny"].with_(
        name="timeout_bm32", T=200, d=256, F=320, E=8, k=3, block_m=32, seed=2106, logits_kind="normal")
    inp = W.make_inputs(cfg)
    lay = DeviceLayer(inp)
    run = (lambda: _layer(lay)) if use_layer else lay.run
    M.moe_debug_timeouts(20_000_000, 1)          # 20 ms, one arrival nothing makes
    run()
    torch.cuda.synchronize()
    assert lay.status() == TIMEOUT, M.status_name(lay.status())
    after = _counters(lay.buf)
    assert after[0] == 0 and after[1] == 0, after[:4]   # grid counters back at rest
    # same call, same workspace, default limit: correct again
    M.moe_debug_timeouts(0, 0)
    lay.buf.status.zero_()
    out = run()
    torch.cuda.synchronize()
    assert lay.status() == 0, M.status_name(lay.status())
    compare_out(_bits(out), _oracle_out(inp), cfg.name)
    c2 = _counters(lay.buf)
    assert c2[0] == 0 and c2[1] == 0


def test_repeated_timeouts_keep_the_workspace_usable():
    cfg = W.CONFIGS["tiny"].with_(name="timeout_rep", T=150, d=192, F=192, E=6, k=2, block_m=64, seed=2107,
                                  logits_kind="normal")
    inp = W.make_inputs(cfg)
    lay = DeviceLayer(inp)
    for _ in range(3):
        M.moe_debug_timeouts(5_000_000, 1)
        lay.run()
        torch.cuda.synchronize()
        assert lay.status() == TIMEOUT
        lay.buf.status.zero_()
    M.moe_debug_timeouts(0, 0)
    out = lay.run()
    torch.cuda.synchronize()
    assert lay.status() == 0
    compare_out(_bits(out), _oracle_out(inp), cfg.name)


def test_grouped_gemm_timeout_drains_then_recovers():
    """block_m = 128 (the token-major grouped GEMMs): the epilogue's first
    accumulator-full wait expects one commit more than the MMA issuer makes;
    it gives up while TMA loads, row gathers and MMAs are still in flight,
    and the kernels drain them and return."""
    cfg = W.CONFIGS["relu2"].with_(name="timeout_tokm", T=333, d=320, F=448, E=5, k=2, block_m=128, seed=2108)
    inp = W.make_inputs(cfg)
    lay = DeviceLayer(inp)
    M.moe_debug_timeouts(20_000_000, 1)
    lay.run()
    torch.cuda.synchronize()
    assert lay.status() == TIMEOUT, M.status_name(lay.status())
    M.moe_debug_timeouts(0, 0)
    lay.buf.status.zero_()
    out = lay.run()
    torch.cuda.synchronize()
    assert lay.status() == 0, M.status_name(lay.status())
    compare_out(_bits(out), _oracle_out(inp), cfg.name)


def test_pair_gemm_timeout_drains_then_recovers():
    """The same on CTA pairs (d, d_ff >= 1024: the paired gate/up and down
    GEMMs, cta_group::2): both CTAs' epilogues give up, the even CTA drains
    the pair's MMAs and its stages' loads, the odd CTA waits for its last
    loads, and the pair frees its tensor memory."""
    cfg = W.CONFIGS["dsv3"].with_(name="timeout_pair", T=600, d=1024, F=1024, seed=2109)
    inp = W.make_inputs(cfg)
    lay = DeviceLayer(inp)
    M.moe_debug_timeouts(20_000_000, 1)
    lay.run()
    torch.cuda.synchronize()
    assert lay.status() == TIMEOUT, M.status_name(lay.status())
    M.moe_debug_timeouts(0, 0)
    lay.buf.status.zero_()
    out = lay.run()
    torch.cuda.synchronize()
    assert lay.status() == 0, M.status_name(lay.status())
    compare_out(_bits(out), _oracle_out(inp), cfg.name)
