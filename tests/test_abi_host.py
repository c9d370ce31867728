"""The C-ABI library loads, exports every entry point include/moe.h declares,
and rejects invalid arguments on the host before touching a GPU.

No call here reaches a CUDA API: each one fails a host check (or is a pure
size query), so the suite runs on machines without a GPU.
"""
import ctypes
import os
import re

import pytest

import oracle
from grouped_gemm_gating_b200 import build as B
from grouped_gemm_gating_b200 import moe as M

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return M.load_library()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)


def test_header_declares_the_abi():
    names = set(declared_functions())
    assert {"moe_route", "moe_align", "moe_forward", "moe_workspace_size", "moe_max_padded",
            "moe_read_status", "moe_align_workspace_size"} <= names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert ctypes.CDLL(M.library_path()) is not None


def test_max_padded_matches_oracle(lib):
    for T, k, E, bm in [(3, 8, 128, 16), (4096, 4, 18, 128), (0, 2, 8, 16), (16384, 8, 128, 128), (256, 6, 128, 16)]:
        assert M.moe_max_padded(T, k, E, bm) == oracle.max_padded(T, k, E, bm)
    assert M.moe_max_padded(3, 8, 128, 48) == -1
    assert M.moe_max_padded(-1, 8, 128, 16) == -1


def test_workspace_sizes(lib):
    T, d, F, E, k, bm = 4096, 3072, 2560, 18, 4, 128
    P = oracle.max_padded(T, k, E, bm) + T  # shared rows (T is a multiple of bm)
    size = M.moe_workspace_size(T, d, F, E, k, bm, M.ACT_SWIGLU, 1)
    counters = 65536
    # counters, h [P_total, F] bf16, fp32 accumulator [T, d], and (d, F >= 1024)
    # the token rows in expert-sorted order [P_total, d] bf16
    assert size >= P * 2 * F + T * 4 * d + P * 2 * d + counters
    assert size <= P * 2 * F + T * 4 * d + P * 2 * d + counters + 1280
    d_small = 512
    size = M.moe_workspace_size(T, d_small, F, E, k, bm, M.ACT_SWIGLU, 1)
    assert P * 2 * F + T * 4 * d_small + counters <= size <= P * 2 * F + T * 4 * d_small + counters + 1024
    # block_m <= 64 keeps h in shared memory: counters and the accumulator only
    small = M.moe_workspace_size(3, 2048, 768, 128, 8, 16, M.ACT_SWIGLU, 0)
    assert 3 * 4 * 2048 + counters <= small <= 3 * 4 * 2048 + counters + 1024
    assert M.moe_workspace_size(T, d + 32, F, E, k, bm, M.ACT_SWIGLU, 0) == 0   # d % 64
    assert M.moe_workspace_size(T, d, F, 300, k, bm, M.ACT_SWIGLU, 0) == 0      # E > 256
    assert M.moe_align_workspace_size(3, 8, 128) == 0                           # single block
    assert M.moe_align_workspace_size(16384, 8, 128) == (131072 // 2048) * 128 * 4


def test_status_strings(lib):
    assert lib.moe_status_string(0) == b"MOE_OK"
    assert lib.moe_status_string(6) == b"MOE_ERR_DEVICE_TIMEOUT"


NULL = None


def test_route_host_checks(lib):
    r = lib.moe_route
    assert r(NULL, 4, 8, 9, 1, 1, 0, 1, 1.0, NULL, NULL, NULL, NULL) == 1      # k > E
    assert r(NULL, 4, 300, 2, 1, 1, 0, 1, 1.0, NULL, NULL, NULL, NULL) == 2    # E > 256
    assert r(NULL, 4, 18, 4, 4, 2, 0, 1, 1.0, NULL, NULL, NULL, NULL) == 1     # E % n_group
    assert r(NULL, 4, 18, 4, 6, 7, 0, 1, 1.0, NULL, NULL, NULL, NULL) == 1     # topk_group > n_group
    assert r(NULL, 4, 18, 7, 6, 2, 0, 1, 1.0, NULL, NULL, NULL, NULL) == 1     # k > topk_group*E/n_group
    assert r(NULL, 4, 18, 4, 6, 4, 5, 1, 1.0, NULL, NULL, NULL, NULL) == 1     # bad group score
    assert r(NULL, 4, 8, 2, 1, 1, 0, 1, 0.0, NULL, NULL, NULL, NULL) == 1      # scaling <= 0
    assert r(NULL, 4, 8, 2, 1, 1, 0, 1, 1.0, NULL, NULL, NULL, NULL) == 1      # null pointers
    assert r(NULL, 0, 8, 2, 1, 1, 0, 1, 1.0, NULL, NULL, NULL, NULL) == 0      # T == 0: no-op


def test_router_host_checks(lib):
    r = lib.moe_router
    #        x     T  d    w_g   E    k  ng tg gs rn scale logits ids   wts   status stream
    assert r(NULL, 4, 128, NULL, 300, 2, 1, 1, 0, 1, 1.0, NULL, NULL, NULL, NULL, NULL) == 2    # E > 256
    assert r(NULL, 4, 128, NULL, 64, 17, 1, 1, 0, 1, 1.0, NULL, NULL, NULL, NULL, NULL) == 2    # k > 16
    assert r(NULL, 4, 96, NULL, 8, 2, 1, 1, 0, 1, 1.0, NULL, NULL, NULL, NULL, NULL) == 2      # d % 64
    assert r(NULL, 4, 128, NULL, 8, 9, 1, 1, 0, 1, 1.0, NULL, NULL, NULL, NULL, NULL) == 1     # k > E
    assert r(NULL, 4, 128, NULL, 18, 4, 4, 2, 0, 1, 1.0, NULL, NULL, NULL, NULL, NULL) == 1    # E % n_group
    assert r(NULL, 4, 128, NULL, 8, 2, 1, 1, 0, 1, 1.0, NULL, NULL, NULL, NULL, NULL) == 1     # null pointers
    assert r(NULL, 0, 128, NULL, 8, 2, 1, 1, 0, 1, 1.0, NULL, NULL, NULL, NULL, NULL) == 0     # T == 0: no-op


def test_align_host_checks(lib):
    a = lib.moe_align
    p = ctypes.c_void_p(16)
    assert a(p, 4, 2, 8, 48, p, p, p, p, NULL, 0, NULL, NULL) == 1             # block_m
    assert a(p, 4, 2, 8, 16, NULL, p, p, p, NULL, 0, NULL, NULL) == 1          # null output
    assert a(p, 16384, 8, 128, 128, p, p, p, p, NULL, 0, NULL, NULL) == 3      # missing workspace
    assert a(p, 16384, 8, 128, 128, p, p, p, p, p, 8, NULL, NULL) == 3         # workspace too small


def test_forward_host_checks(lib):
    f = lib.moe_forward
    p = ctypes.c_void_p(256)
    odd = ctypes.c_void_p(258)
    args = lambda **kw: [kw.get("x", p), kw.get("T", 4), kw.get("d", 128), p, p, kw.get("E", 8), kw.get("F", 128),
                         kw.get("w13s", NULL), kw.get("w2s", NULL), kw.get("ns", 0), p, kw.get("k", 2), p, p, p, p,
                         kw.get("bm", 16), kw.get("act", 0), p, kw.get("ws", p), kw.get("wsb", 1 << 40), NULL, NULL]
    assert f(*args(d=96)) == 2                 # d % 64
    assert f(*args(F=100)) == 2                # F % 64
    assert f(*args(E=257)) == 2                # E > 256
    assert f(*args(k=9, E=8)) == 1             # k > E
    assert f(*args(bm=8)) == 2                 # block_m
    assert f(*args(act=3)) == 1                # activation
    assert f(*args(ns=1)) == 1                 # shared expert weights missing
    assert f(*args(x=odd)) == 1                # misaligned
    assert f(*args(x=NULL)) == 1               # null
    assert f(*args(wsb=16)) == 3               # workspace too small
    assert f(*args(ws=NULL)) == 3              # workspace missing
    assert f(*args(T=0, x=NULL)) == 0          # T == 0: no-op


def test_backward_host_checks(lib):
    f = lib.moe_backward
    p = ctypes.c_void_p(256)
    odd = ctypes.c_void_p(258)
    args = lambda **kw: [kw.get("x", p), kw.get("T", 4), kw.get("d", 128), p, p, kw.get("E", 8), kw.get("F", 128),
                         kw.get("w13s", NULL), kw.get("w2s", NULL), kw.get("ns", 0), p, kw.get("k", 2), p, p, p,
                         kw.get("act", 0), kw.get("dout", p), kw.get("dx", p), kw.get("dw13", p), p, NULL, NULL,
                         kw.get("dtopk", NULL), kw.get("ws", p), kw.get("wsb", 1 << 40), NULL, NULL]
    assert f(*args(d=96)) == 2                 # d % 64
    assert f(*args(F=100)) == 2                # F % 64
    assert f(*args(E=257)) == 2                # E > 256
    assert f(*args(k=9, E=8)) == 1             # k > E
    assert f(*args(act=3)) == 1                # activation
    assert f(*args(ns=1)) == 1                 # shared expert weights / gradients missing
    assert f(*args(dout=odd)) == 1             # misaligned
    assert f(*args(dtopk=ctypes.c_void_p(260))) == 1   # dL/dw must be 16-byte aligned
    assert f(*args(dw13=NULL)) == 1            # gradient output missing
    assert f(*args(dx=NULL)) == 1
    assert f(*args(wsb=16)) == 3               # workspace too small
    assert f(*args(ws=NULL)) == 3              # workspace missing
    T, d, F, E, k = 300, 256, 192, 8, 2
    P = oracle.max_padded(T, k, E, 128)
    need = M.moe_backward_workspace_size(T, d, F, E, k, M.ACT_SWIGLU, 0)
    # x and dL/dout rows [P, d] bf16 each, fp32 pre-activations and bf16 da [P, 2F], w*h [P, F], fp32 dx [T, d]
    lo = P * (2 * d * 2 + 2 * F * 4 + 2 * F * 2 + F * 2) + T * d * 4
    assert lo <= need <= lo + 1792
    assert M.moe_backward_workspace_size(T, d, 100, E, k, M.ACT_SWIGLU, 0) == 0


def test_layer_host_checks(lib):
    f = lib.moe_layer
    p = ctypes.c_void_p(256)
    odd = ctypes.c_void_p(258)

    def args(**kw):
        return [kw.get("logits", p), kw.get("T", 4), kw.get("E", 8), kw.get("k", 2), kw.get("ng", 1), kw.get("tg", 1),
                0, 1, kw.get("scale", 1.0), kw.get("x", p), kw.get("d", 128), p, p, kw.get("F", 128), NULL, NULL,
                kw.get("ns", 0), kw.get("bm", 16), kw.get("act", 0), p, p, p, p, p, kw.get("inv", p), p,
                kw.get("ws", p), kw.get("wsb", 1 << 40), NULL, NULL]
    assert f(*args(k=9)) == 1                  # k > E
    assert f(*args(ng=3)) == 1                 # E % n_group
    assert f(*args(scale=0.0)) == 1            # routed_scaling <= 0
    assert f(*args(d=96)) == 2                 # d % 64
    assert f(*args(bm=8)) == 2                 # block_m
    assert f(*args(act=3)) == 1                # activation
    assert f(*args(ns=1)) == 1                 # shared expert weights missing
    assert f(*args(x=odd)) == 1                # misaligned
    assert f(*args(logits=NULL)) == 1          # null logits
    assert f(*args(inv=NULL)) == 1             # inv_pos is an output here
    assert f(*args(wsb=16)) == 3               # workspace too small
    assert f(*args(T=0, x=NULL, logits=NULL)) == 0  # T == 0: no-op


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(M, "_lib", None)
    monkeypatch.setattr(M, "library_path", lambda: str(tmp_path / "nope.so"))
    with pytest.raises(RuntimeError, match="missing"):
        M.load_library()
