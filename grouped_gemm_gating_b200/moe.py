"""Python binding of the C ABI in include/moe.h (argument marshalling only).

Every function here passes device pointers, sizes and the current CUDA
stream of torch to the shared library ``libmoe_b200.so`` and raises
:class:`MoEError` when the library returns an error.  All computation runs
in the library's CUDA kernels; there is no CPU fallback.  If the library has
not been built, the first call raises immediately.

torch is used only for device memory (tensors as buffers) and streams.
bf16 tensors are passed as their raw 16-bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import build as _build

ACT_SWIGLU = 0
ACT_RELU2 = 1
GROUP_MAX = 0
GROUP_TOP2SUM = 1

_STATUS = {
    0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
    4: "MOE_ERR_CUDA", 5: "MOE_ERR_NONFINITE", 6: "MOE_ERR_DEVICE_TIMEOUT", 7: "MOE_ERR_BAD_EXPERT_ID",
}

# name -> (restype, argtypes)
_P = ctypes.c_void_p
_I = ctypes.c_int
_SIG = {
    "moe_max_padded": (ctypes.c_int64, [_I, _I, _I, _I]),
    "moe_align_workspace_size": (ctypes.c_size_t, [_I, _I, _I]),
    "moe_workspace_size": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "moe_route": (_I, [_P, _I, _I, _I, _I, _I, _I, _I, ctypes.c_float, _P, _P, _P, _P]),
    "moe_router": (_I, [_P, _I, _I, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float, _P, _P, _P, _P, _P]),
    "moe_align": (_I, [_P, _I, _I, _I, _I, _P, _P, _P, _P, _P, ctypes.c_size_t, _P, _P]),
    "moe_align_noalloc": (_I, [_P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "moe_route_align": (_I, [_P, _I, _I, _I, _I, _I, _I, _I, ctypes.c_float, _I, _P, _P, _P, _P, _P, _P, _P,
                             ctypes.c_size_t, _P, _P]),
    "moe_forward": (_I, [_P, _I, _I, _P, _P, _I, _I, _P, _P, _I, _P, _I, _P, _P, _P, _P, _I, _I,
                         _P, _P, ctypes.c_size_t, _P, _P]),
    "moe_layer": (_I, [_P, _I, _I, _I, _I, _I, _I, _I, ctypes.c_float, _P, _I, _P, _P, _I, _P, _P, _I, _I, _I,
                       _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P, _P]),
    "moe_backward_workspace_size": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I, _I]),
    "moe_backward": (_I, [_P, _I, _I, _P, _P, _I, _I, _P, _P, _I, _P, _I, _P, _P, _P, _I, _P, _P, _P, _P, _P, _P,
                          _P, _P, ctypes.c_size_t, _P, _P]),
    "moe_forward_fp8": (_I, [_P, _I, _I, _P, _P, _P, _P, _I, _I, _P, _P, _P, _P, _I, _P, _I, _P, _P, _P, _P, _I,
                             _I, _P, _P, ctypes.c_size_t, _P, _P]),
    "moe_layer_fp8": (_I, [_P, _I, _I, _I, _I, _I, _I, _I, ctypes.c_float, _P, _I, _P, _P, _P, _P, _I, _P, _P, _P,
                           _P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P, _P]),
    "moe_read_status": (_I, [_P, _P]),
    "moe_status_string": (ctypes.c_char_p, [_I]),
    "moe_last_launch_count": (_I, []),
    "moe_debug_timeouts": (_I, [ctypes.c_uint64, _I]),
    "moe_profile_enable": (_I, [_I]),
    "moe_profile_collect": (_I, [_P, _P, _I, _I]),
}

STAGES = ("route", "align", "gate_up_gemm", "down_gemm", "combine", "route_align", "fused_expert", "permute",
          "router", "bwd_recompute", "bwd_dh_gemm", "bwd_dx_gemm", "bwd_dw13_gemm", "bwd_dw2_gemm")

_lib = None
_lock = threading.Lock()


class MoEError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {_STATUS.get(code, code)}")


def library_path() -> str:
    return _build.LIB_PATH


def load_library():
    """Load libmoe_b200.so (raising if it was not built) and bind signatures."""
    global _lib
    with _lock:
        if _lib is None:
            path = library_path()
            if not os.path.exists(path):
                raise RuntimeError(
                    f"CUDA library {path} is missing: build it with "
                    "`python -m grouped_gemm_gating_b200.build` (nvcc, sm_100a)")
            lib = ctypes.CDLL(path)
            for name, (res, args) in _SIG.items():
                f = getattr(lib, name)
                f.restype = res
                f.argtypes = args
            _lib = lib
    return _lib


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(device=None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(fn, code):
    if code != 0:
        raise MoEError(fn, code)


def _bits(t):
    """bf16 tensor -> the same storage viewed as int16 patterns (checked)."""
    if t is None:
        return None
    if t.dtype != torch.bfloat16:
        raise ValueError("expected a bfloat16 tensor")
    return t


# ---------------------------------------------------------------- sizes ---

def moe_max_padded(T, k, E, block_m) -> int:
    return int(load_library().moe_max_padded(T, k, E, block_m))


def moe_align_workspace_size(T, k, E) -> int:
    return int(load_library().moe_align_workspace_size(T, k, E))


def moe_workspace_size(T, d, F, E, k, block_m, act, n_shared) -> int:
    return int(load_library().moe_workspace_size(T, d, F, E, k, block_m, act, n_shared))


def moe_last_launch_count() -> int:
    return int(load_library().moe_last_launch_count())


def moe_debug_timeouts(wait_limit_ns: int = 0, unreachable_arrivals: int = 0) -> None:
    """Test hook: the wait limit of kernels launched afterwards (0: the
    default 2 s) and, when unreachable_arrivals > 0, a start barrier in the
    fused expert kernel that waits for more CTAs than its grid has."""
    _check("moe_debug_timeouts", load_library().moe_debug_timeouts(int(wait_limit_ns), int(unreachable_arrivals)))


def moe_profile_enable(on: bool = True) -> None:
    """Start (or stop) recording CUDA events around every kernel launch."""
    _check("moe_profile_enable", load_library().moe_profile_enable(1 if on else 0))


def moe_profile_collect(release: bool = True) -> dict:
    """Summed milliseconds and launch counts per stage of the recorded events.

    release=False keeps the records (read a captured graph's events again
    after its next replay)."""
    n = len(STAGES)
    ms = (ctypes.c_double * n)()
    calls = (ctypes.c_int * n)()
    _check("moe_profile_collect", load_library().moe_profile_collect(ms, calls, n, 1 if release else 0))
    return {name: (float(ms[i]), int(calls[i])) for i, name in enumerate(STAGES)}


# ---------------------------------------------------------------- calls ---

def moe_route(logits, k, topk_ids, topk_weights, n_group=1, topk_group=1, group_score=GROUP_MAX,
              renormalize=True, routed_scaling=1.0, dev_status=None):
    """Top-k gating: fills topk_ids [T,k] int32 and topk_weights [T,k] fp32."""
    T, E = logits.shape
    if logits.dtype != torch.float32 or topk_ids.dtype != torch.int32 or topk_weights.dtype != torch.float32:
        raise ValueError("moe_route: logits/weights fp32, ids int32")
    code = load_library().moe_route(_ptr(logits), T, E, k, n_group, topk_group, group_score,
                                    1 if renormalize else 0, float(routed_scaling),
                                    _ptr(topk_ids), _ptr(topk_weights), _ptr(dev_status),
                                    _stream(logits.device))
    _check("moe_route", code)


def moe_router(x, w_gate, k, logits, topk_ids, topk_weights, n_group=1, topk_group=1, group_score=GROUP_MAX,
               renormalize=True, routed_scaling=1.0, dev_status=None):
    """Router projection x . W_g^T (fp32 logits [T, E]) and top-k gating in one call."""
    T, d = x.shape
    E = w_gate.shape[0]
    if w_gate.shape[1] != d:
        raise ValueError("moe_router: w_gate must be [E, d]")
    if logits.dtype != torch.float32 or topk_weights.dtype != torch.float32 or topk_ids.dtype != torch.int32:
        raise ValueError("moe_router: logits/weights fp32, ids int32")
    code = load_library().moe_router(_ptr(_bits(x)), T, d, _ptr(_bits(w_gate)), E, k, n_group, topk_group,
                                     group_score, 1 if renormalize else 0, float(routed_scaling), _ptr(logits),
                                     _ptr(topk_ids), _ptr(topk_weights), _ptr(dev_status), _stream(x.device))
    _check("moe_router", code)


def moe_align(topk_ids, E, block_m, sorted_token_ids, expert_ids, num_tokens_post_padded, inv_pos,
              ws=None, dev_status=None):
    """Sort slots by expert and pad to block_m (outputs preallocated)."""
    T, k = topk_ids.shape
    for t in (topk_ids, sorted_token_ids, expert_ids, num_tokens_post_padded, inv_pos):
        if t.dtype != torch.int32:
            raise ValueError("moe_align: int32 tensors expected")
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    code = load_library().moe_align(_ptr(topk_ids), T, k, E, block_m, _ptr(sorted_token_ids),
                                    _ptr(expert_ids), _ptr(num_tokens_post_padded), _ptr(inv_pos),
                                    _ptr(ws), ws_bytes, _ptr(dev_status), _stream(topk_ids.device))
    _check("moe_align", code)


def moe_route_align(logits, k, block_m, topk_ids, topk_weights, sorted_token_ids, expert_ids,
                    num_tokens_post_padded, inv_pos, ws=None, n_group=1, topk_group=1, group_score=GROUP_MAX,
                    renormalize=True, routed_scaling=1.0, dev_status=None):
    """moe_route then moe_align in one call (one kernel for small batches)."""
    T, E = logits.shape
    if logits.dtype != torch.float32 or topk_weights.dtype != torch.float32:
        raise ValueError("moe_route_align: logits/weights fp32")
    for t in (topk_ids, sorted_token_ids, expert_ids, num_tokens_post_padded, inv_pos):
        if t.dtype != torch.int32:
            raise ValueError("moe_route_align: int32 index tensors expected")
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    code = load_library().moe_route_align(
        _ptr(logits), T, E, k, n_group, topk_group, group_score, 1 if renormalize else 0,
        float(routed_scaling), block_m, _ptr(topk_ids), _ptr(topk_weights), _ptr(sorted_token_ids),
        _ptr(expert_ids), _ptr(num_tokens_post_padded), _ptr(inv_pos), _ptr(ws), ws_bytes,
        _ptr(dev_status), _stream(logits.device))
    _check("moe_route_align", code)


def moe_align_noalloc(topk_ids, E, block_m, sorted_token_ids, expert_ids, num_tokens_post_padded,
                      inv_pos, dev_status=None):
    """moe_align without a workspace, for callers that cannot allocate device
    memory: the library keeps the scratch in a fixed static device array
    (limit ceil(T*k/2048)*E <= 131072).  Calls that overlap on the GPU race
    on that array."""
    T, k = topk_ids.shape
    for t in (topk_ids, sorted_token_ids, expert_ids, num_tokens_post_padded, inv_pos):
        if t.dtype != torch.int32:
            raise ValueError("moe_align_noalloc: int32 tensors expected")
    code = load_library().moe_align_noalloc(_ptr(topk_ids), T, k, E, block_m, _ptr(sorted_token_ids),
                                            _ptr(expert_ids), _ptr(num_tokens_post_padded), _ptr(inv_pos),
                                            _ptr(dev_status), _stream(topk_ids.device))
    _check("moe_align_noalloc", code)


def moe_forward(x, w13, w2, topk_weights, sorted_token_ids, expert_ids, num_tokens_post_padded,
                inv_pos, block_m, act, out, ws, w13_shared=None, w2_shared=None, dev_status=None):
    """Grouped expert GEMMs + weighted scatter-reduce into out [T, d] bf16."""
    T, d = x.shape
    E, n1, _ = w13.shape
    F = w2.shape[2]
    k = topk_weights.shape[1] if topk_weights.dim() == 2 else 1
    n_shared = 0 if w13_shared is None else 1
    code = load_library().moe_forward(
        _ptr(_bits(x)), T, d, _ptr(_bits(w13)), _ptr(_bits(w2)), E, F,
        _ptr(_bits(w13_shared)), _ptr(_bits(w2_shared)), n_shared,
        _ptr(topk_weights), k, _ptr(sorted_token_ids), _ptr(expert_ids),
        _ptr(num_tokens_post_padded), _ptr(inv_pos), block_m, act,
        _ptr(_bits(out)), _ptr(ws), ws.numel() * ws.element_size(), _ptr(dev_status),
        _stream(x.device))
    _check("moe_forward", code)


def moe_layer(logits, x, w13, w2, k, block_m, act, topk_ids, topk_weights, sorted_token_ids, expert_ids,
              num_tokens_post_padded, inv_pos, out, ws, w13_shared=None, w2_shared=None, n_group=1, topk_group=1,
              group_score=GROUP_MAX, renormalize=True, routed_scaling=1.0, dev_status=None):
    """Route, align and forward in one call (one kernel for decode batches)."""
    T, E = logits.shape
    d = x.shape[1]
    F = w2.shape[2]
    if logits.dtype != torch.float32 or topk_weights.dtype != torch.float32:
        raise ValueError("moe_layer: logits/weights fp32")
    n_shared = 0 if w13_shared is None else 1
    code = load_library().moe_layer(
        _ptr(logits), T, E, k, n_group, topk_group, group_score, 1 if renormalize else 0, float(routed_scaling),
        _ptr(_bits(x)), d, _ptr(_bits(w13)), _ptr(_bits(w2)), F, _ptr(_bits(w13_shared)), _ptr(_bits(w2_shared)),
        n_shared, block_m, act, _ptr(topk_ids), _ptr(topk_weights), _ptr(sorted_token_ids), _ptr(expert_ids),
        _ptr(num_tokens_post_padded), _ptr(inv_pos), _ptr(_bits(out)), _ptr(ws), ws.numel() * ws.element_size(),
        _ptr(dev_status), _stream(x.device))
    _check("moe_layer", code)


def moe_backward_workspace_size(T, d, F, E, k, act, n_shared) -> int:
    return int(load_library().moe_backward_workspace_size(T, d, F, E, k, act, n_shared))


def moe_backward(x, w13, w2, topk_weights, sorted_token_ids, expert_ids, num_tokens_post_padded, act, dout,
                 dx, dw13, dw2, ws, w13_shared=None, w2_shared=None, dw13_shared=None, dw2_shared=None,
                 dtopk_weights=None, dev_status=None):
    """The layer's backward (align outputs for block_m = 128): fills dx [T, d],
    dw13 [E, n1, d], dw2 [E, d, F] (bf16) and, when given, dtopk_weights [T, k]
    fp32 and the shared expert's weight gradients."""
    T, d = x.shape
    E, n1, _ = w13.shape
    F = w2.shape[2]
    k = topk_weights.shape[1] if topk_weights.dim() == 2 else 1
    n_shared = 0 if w13_shared is None else 1
    if dtopk_weights is not None and dtopk_weights.dtype != torch.float32:
        raise ValueError("moe_backward: dtopk_weights must be fp32")
    code = load_library().moe_backward(
        _ptr(_bits(x)), T, d, _ptr(_bits(w13)), _ptr(_bits(w2)), E, F, _ptr(_bits(w13_shared)),
        _ptr(_bits(w2_shared)), n_shared, _ptr(topk_weights), k, _ptr(sorted_token_ids), _ptr(expert_ids),
        _ptr(num_tokens_post_padded), act, _ptr(_bits(dout)), _ptr(_bits(dx)), _ptr(_bits(dw13)), _ptr(_bits(dw2)),
        _ptr(_bits(dw13_shared)), _ptr(_bits(dw2_shared)), _ptr(dtopk_weights), _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(dev_status), _stream(x.device))
    _check("moe_backward", code)


class MoEGradBuffers:
    """Device buffers of one layer shape's backward (plumbing only): the
    gradients and the backward's workspace, allocated once."""

    def __init__(self, T, d, F, E, k, act=ACT_SWIGLU, n_shared=0, device="cuda"):
        dev = torch.device(device)
        n1 = 2 * F if act == ACT_SWIGLU else F
        self.act, self.n_shared = act, n_shared
        bf = dict(dtype=torch.bfloat16, device=dev)
        self.dx = torch.empty((T, d), **bf)
        self.dw13 = torch.empty((E, n1, d), **bf)
        self.dw2 = torch.empty((E, d, F), **bf)
        self.dw13_shared = torch.empty((1, n1, d), **bf) if n_shared else None
        self.dw2_shared = torch.empty((1, d, F), **bf) if n_shared else None
        self.dtopk = torch.empty((T, k), dtype=torch.float32, device=dev)
        n = moe_backward_workspace_size(T, d, F, E, k, act, n_shared)
        if n == 0:
            raise ValueError("unsupported layer shape")
        self.ws = torch.empty(n, dtype=torch.uint8, device=dev)

    def backward(self, fwd: "MoEBuffers", x, w13, w2, dout, w13_shared=None, w2_shared=None):
        """Gradients of the layer whose routing and align outputs fwd holds
        (block_m = 128)."""
        moe_backward(x, w13, w2, fwd.topk_weights, fwd.sorted_token_ids, fwd.expert_ids, fwd.ntpp, self.act,
                     dout, self.dx, self.dw13, self.dw2, self.ws, w13_shared, w2_shared, self.dw13_shared,
                     self.dw2_shared, self.dtopk, fwd.status)


class Fp8Experts:
    """fp8 expert weights on the device (plumbing): e4m3 bytes and the
    K-block-major power-of-two scale bytes of w13 and w2 (and of the shared
    expert), as uint8 tensors in the layouts include/moe.h gives."""

    def __init__(self, w13_q, w13_s, w2_q, w2_s, w13s_q=None, w13s_s=None, w2s_q=None, w2s_s=None):
        for t in (w13_q, w13_s, w2_q, w2_s):
            if t.dtype != torch.uint8:
                raise ValueError("fp8 weights and scales are uint8 tensors")
        self.w13_q, self.w13_s, self.w2_q, self.w2_s = w13_q, w13_s, w2_q, w2_s
        self.w13s_q, self.w13s_s, self.w2s_q, self.w2s_s = w13s_q, w13s_s, w2s_q, w2s_s
        self.E, self.n1, self.d = w13_q.shape
        self.F = w2_q.shape[2]
        self.n_shared = 0 if w13s_q is None else 1


def moe_forward_fp8(x, wq: Fp8Experts, topk_weights, sorted_token_ids, expert_ids, num_tokens_post_padded,
                    inv_pos, block_m, act, out, ws, dev_status=None):
    """moe_forward with fp8 expert weights (block_m 16, 32 or 64)."""
    T, d = x.shape
    k = topk_weights.shape[1] if topk_weights.dim() == 2 else 1
    code = load_library().moe_forward_fp8(
        _ptr(_bits(x)), T, d, _ptr(wq.w13_q), _ptr(wq.w13_s), _ptr(wq.w2_q), _ptr(wq.w2_s), wq.E, wq.F,
        _ptr(wq.w13s_q), _ptr(wq.w13s_s), _ptr(wq.w2s_q), _ptr(wq.w2s_s), wq.n_shared, _ptr(topk_weights), k,
        _ptr(sorted_token_ids), _ptr(expert_ids), _ptr(num_tokens_post_padded), _ptr(inv_pos), block_m, act,
        _ptr(_bits(out)), _ptr(ws), ws.numel() * ws.element_size(), _ptr(dev_status), _stream(x.device))
    _check("moe_forward_fp8", code)


def moe_layer_fp8(logits, x, wq: Fp8Experts, k, block_m, act, topk_ids, topk_weights, sorted_token_ids, expert_ids,
                  num_tokens_post_padded, inv_pos, out, ws, n_group=1, topk_group=1, group_score=GROUP_MAX,
                  renormalize=True, routed_scaling=1.0, dev_status=None):
    """moe_layer with fp8 expert weights (one launch for decode batches)."""
    T, E = logits.shape
    code = load_library().moe_layer_fp8(
        _ptr(logits), T, E, k, n_group, topk_group, group_score, 1 if renormalize else 0, float(routed_scaling),
        _ptr(_bits(x)), wq.d, _ptr(wq.w13_q), _ptr(wq.w13_s), _ptr(wq.w2_q), _ptr(wq.w2_s), wq.F, _ptr(wq.w13s_q),
        _ptr(wq.w13s_s), _ptr(wq.w2s_q), _ptr(wq.w2s_s), wq.n_shared, block_m, act, _ptr(topk_ids),
        _ptr(topk_weights), _ptr(sorted_token_ids), _ptr(expert_ids), _ptr(num_tokens_post_padded), _ptr(inv_pos),
        _ptr(_bits(out)), _ptr(ws), ws.numel() * ws.element_size(), _ptr(dev_status), _stream(x.device))
    _check("moe_layer_fp8", code)


def moe_read_status(dev_status) -> int:
    """Synchronise the current stream and return the device status code."""
    return int(load_library().moe_read_status(_ptr(dev_status), _stream(dev_status.device)))


def status_name(code: int) -> str:
    return _STATUS.get(code, str(code))


# ------------------------------------------------------------ buffers -----

class MoEBuffers:
    """Device buffers of one layer shape, allocated once (plumbing only).

    Holds the routing outputs, the align outputs, both workspaces, the output
    and a status word, so that a step is three library calls with no
    allocation: :meth:`route`, :meth:`align`, :meth:`forward`.
    """

    def __init__(self, T, d, F, E, k, block_m, act=ACT_SWIGLU, n_shared=0, device="cuda"):
        self.T, self.d, self.F, self.E, self.k = T, d, F, E, k
        self.block_m, self.act, self.n_shared = block_m, act, n_shared
        dev = torch.device(device)
        P = moe_max_padded(T, k, E, block_m)
        if P < 0:
            raise ValueError("invalid layer shape")
        self.P_max = P
        i32 = dict(dtype=torch.int32, device=dev)
        self.topk_ids = torch.empty((T, k), **i32)
        self.topk_weights = torch.empty((T, k), dtype=torch.float32, device=dev)
        self.sorted_token_ids = torch.empty(P, **i32)
        self.expert_ids = torch.empty(P // block_m, **i32)
        self.ntpp = torch.empty(1, **i32)
        self.inv_pos = torch.empty(max(T * k, 1), **i32)
        aws = moe_align_workspace_size(T, k, E)
        self.align_ws = torch.empty(max(aws // 4, 1), **i32) if aws else None
        fws = moe_workspace_size(T, d, F, E, k, block_m, act, n_shared)
        if fws == 0:
            raise ValueError("unsupported layer shape")
        # zero-filled: the workspace's leading counter block must start at zero
        self.ws = torch.zeros(fws, dtype=torch.uint8, device=dev)
        self.out = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
        self.status = torch.zeros(1, **i32)

    def route(self, logits, n_group=1, topk_group=1, group_score=GROUP_MAX, renormalize=True,
              routed_scaling=1.0):
        moe_route(logits, self.k, self.topk_ids, self.topk_weights, n_group, topk_group, group_score,
                  renormalize, routed_scaling, self.status)

    def align(self):
        moe_align(self.topk_ids, self.E, self.block_m, self.sorted_token_ids, self.expert_ids,
                  self.ntpp, self.inv_pos, self.align_ws, self.status)

    def route_align(self, logits, n_group=1, topk_group=1, group_score=GROUP_MAX, renormalize=True,
                    routed_scaling=1.0):
        moe_route_align(logits, self.k, self.block_m, self.topk_ids, self.topk_weights, self.sorted_token_ids,
                        self.expert_ids, self.ntpp, self.inv_pos, self.align_ws, n_group, topk_group, group_score,
                        renormalize, routed_scaling, self.status)

    def layer(self, logits, x, w13, w2, w13_shared=None, w2_shared=None, n_group=1, topk_group=1,
              group_score=GROUP_MAX, renormalize=True, routed_scaling=1.0):
        moe_layer(logits, x, w13, w2, self.k, self.block_m, self.act, self.topk_ids, self.topk_weights,
                  self.sorted_token_ids, self.expert_ids, self.ntpp, self.inv_pos, self.out, self.ws, w13_shared,
                  w2_shared, n_group, topk_group, group_score, renormalize, routed_scaling, self.status)
        return self.out

    def layer_fp8(self, logits, x, wq: "Fp8Experts", n_group=1, topk_group=1, group_score=GROUP_MAX,
                  renormalize=True, routed_scaling=1.0):
        moe_layer_fp8(logits, x, wq, self.k, self.block_m, self.act, self.topk_ids, self.topk_weights,
                      self.sorted_token_ids, self.expert_ids, self.ntpp, self.inv_pos, self.out, self.ws, n_group,
                      topk_group, group_score, renormalize, routed_scaling, self.status)
        return self.out

    def forward_fp8(self, x, wq: "Fp8Experts"):
        moe_forward_fp8(x, wq, self.topk_weights, self.sorted_token_ids, self.expert_ids, self.ntpp, self.inv_pos,
                        self.block_m, self.act, self.out, self.ws, self.status)
        return self.out

    def forward(self, x, w13, w2, w13_shared=None, w2_shared=None):
        moe_forward(x, w13, w2, self.topk_weights, self.sorted_token_ids, self.expert_ids, self.ntpp,
                    self.inv_pos, self.block_m, self.act, self.out, self.ws, w13_shared, w2_shared,
                    self.status)
        return self.out
