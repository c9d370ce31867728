"""The allocation-free align entry point against the workspace one.

moe_align_noalloc serves callers that cannot call cudaMalloc (a runtime
that reserves all device memory up front, code running under CUDA graph
capture, a plugin whose host framework owns every allocation).  It keeps
its scratch in a static device array shared by all calls, so the check runs
two different problems back to back through the C ABI and compares each with
moe_align (with a workspace) bit for bit.  This file sorts last so that a
run stopping at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from grouped_gemm_gating_b200 import moe as M
from grouped_gemm_gating_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _outputs(T, k, E, bm):
    P = M.moe_max_padded(T, k, E, bm)
    i32 = dict(dtype=torch.int32, device="cuda")
    return (torch.full((P,), -7, **i32), torch.full((P // bm,), -7, **i32), torch.full((1,), -7, **i32),
            torch.full((max(T * k, 1),), -7, **i32))


def _with_workspace(ids, E, bm):
    T, k = ids.shape
    outs = _outputs(T, k, E, bm)
    n = M.moe_align_workspace_size(T, k, E)
    ws = torch.empty(max(n // 4, 1), dtype=torch.int32, device="cuda") if n else None
    M.moe_align(ids, E, bm, *outs, ws=ws)
    return [o.cpu().numpy() for o in outs]


def _no_alloc(ids, E, bm, status):
    T, k = ids.shape
    outs = _outputs(T, k, E, bm)
    M.moe_align_noalloc(ids, E, bm, *outs, dev_status=status)
    return [o.cpu().numpy() for o in outs]


# the first case fills the static scratch exactly: ceil(T*k / 2048) * E =
# 2048 * 128 = 262144 chunk x expert entries
@pytest.mark.parametrize("T,E,k,bm", [(524288, 128, 8, 128), (16384, 128, 8, 128), (9000, 64, 2, 16),
                                      (5000, 256, 8, 64), (3, 128, 8, 16)])
def test_noalloc_align_matches_workspace_align_twice(T, E, k, bm):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call, seed in enumerate((T + E, T + E + 1)):
        ids = torch.from_numpy(W.random_topk_ids(T, E, k, seed=seed, skew=4.0 * call)).cuda()
        ref = _with_workspace(ids, E, bm)
        got = _no_alloc(ids, E, bm, status)
        assert M.moe_read_status(status) == 0
        for name, a, b in zip(("sorted_token_ids", "expert_ids", "num_tokens_post_padded", "inv_pos"), got, ref):
            assert np.array_equal(a, b), f"call {call}: {name} differs"


@pytest.mark.parametrize("T,k,E", [((1 << 19) + 1, 8, 128),   # one slot past the limit: 2049 * 128 entries
                                   (1 << 18, 16, 256)])       # ceil(T*k/2048) * E = 524288 > 262144
def test_noalloc_align_rejects_sizes_beyond_the_static_scratch(T, k, E):
    ids = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    lib = M.load_library()
    p = ids.data_ptr()
    code = lib.moe_align_noalloc(p, T, k, E, 128, p, p, p, p, None, None)
    assert code == 2, M.status_name(code)   # MOE_ERR_UNSUPPORTED, nothing launched
