"""Seeded synthetic inputs for the fused MoE expert layer.

This module only draws random numbers and packs them into arrays.  It holds
none of the layer's arithmetic (no routing, sorting, GEMM or activation), so
that the CUDA path and the CPU oracle can both be fed from it without sharing
any of the computation they are compared on.

Every tensor is drawn on the host with numpy's PCG64 from a SeedSequence
rooted at ``1000 + config number`` and spawned per tensor (and per expert for
the weight stacks, so the big stacks can be drawn by several threads).  Floats
are drawn in fp32 and rounded to bf16 with round-to-nearest-even; bf16 tensors
are carried as ``uint16`` bit patterns so that the same bits go to the GPU and
to the oracle.

Workload shapes follow the five configurations of the fused MoE layer:

* ``tiny``     T=32,    d=128,  F=256,  E=8,   k=2, SwiGLU, block_m=16
* ``decode``   T=3,     d=2048, F=768,  E=128, k=8, SwiGLU, block_m=16
* ``dsv3``     T=4096,  d=3072, F=2560, E=18 (+1 shared), k=4, n_group=6,
               topk_group=4, SwiGLU, block_m=128
* ``relu2``    T=256,   d=2688, F=1856, E=128, k=6, squared ReLU, block_m=16
* ``zipf``     T=16384, d=2048, F=768,  E=128, k=8, SwiGLU, block_m=128

The model sizes come from the DeepSeek-V3 benchmark builder of the axolotl
vendor-moe diff (scripts/benchmarks/build_deepseek_v3_8b.py, ``build_config``:
hidden 3072, moe_intermediate 2560, 18 routed experts, top-4, n_group 6,
topk_group 4, one shared expert) and from the squared-ReLU expert of the
mlxcel PR "perf(moe): preserve squared-ReLU fused MoE kernel behind a
dedicated flag" (fc1 -> relu^2 -> fc2, no gate).
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor

import numpy as np

ACT_SWIGLU = 0
ACT_RELU2 = 1


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    d: int
    F: int
    E: int
    k: int
    act: int = ACT_SWIGLU
    block_m: int = 16
    n_group: int = 1
    topk_group: int = 1
    group_score: int = 0          # 0 = max logit of the group, 1 = sum of top-2
    renormalize: int = 1
    routed_scaling: float = 1.0
    n_shared: int = 0
    seed: int = 1000
    logits_kind: str = "normal"   # normal | router | uniform | decode_hot | zipf

    @property
    def n1(self) -> int:
        """Rows of the fused first-layer weight per expert (gate+up or fc1)."""
        return 2 * self.F if self.act == ACT_SWIGLU else self.F

    def flops_routed(self) -> int:
        """Algorithmic FLOPs of the routed experts: 2*T*k*(3 or 2)*d*F."""
        mats = 3 if self.act == ACT_SWIGLU else 2
        return 2 * self.T * self.k * mats * self.d * self.F

    def flops_total(self) -> int:
        mats = 3 if self.act == ACT_SWIGLU else 2
        return self.flops_routed() + 2 * self.T * self.n_shared * mats * self.d * self.F

    def with_(self, **kw) -> "MoEConfig":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    "tiny": MoEConfig("tiny", T=32, d=128, F=256, E=8, k=2, block_m=16,
                      seed=1001, logits_kind="router"),
    "decode": MoEConfig("decode", T=3, d=2048, F=768, E=128, k=8, block_m=16,
                        seed=1002, logits_kind="decode_hot"),
    "dsv3": MoEConfig("dsv3", T=4096, d=3072, F=2560, E=18, k=4, block_m=128,
                      n_group=6, topk_group=4, routed_scaling=1.0, n_shared=1,
                      seed=1003, logits_kind="uniform"),
    "relu2": MoEConfig("relu2", T=256, d=2688, F=1856, E=128, k=6, act=ACT_RELU2,
                       block_m=16, seed=1004, logits_kind="normal"),
    "zipf": MoEConfig("zipf", T=16384, d=2048, F=768, E=128, k=8, block_m=128,
                      seed=1005, logits_kind="zipf"),
}


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round to nearest, ties to even); return uint16 bits."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal_bf16(ss: np.random.SeedSequence, shape, std: float) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(ss))
    v = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        v *= np.float32(std)
    return f32_to_bf16_bits(v)


def _stack_normal_bf16(ss: np.random.SeedSequence, n: int, shape, std: float,
                       threads: int = 8) -> np.ndarray:
    """[n, *shape] bf16 stack; one child stream per slice, drawn in parallel."""
    children = ss.spawn(n)
    out = np.empty((n,) + tuple(shape), dtype=np.uint16)

    def fill(i):
        out[i] = _normal_bf16(children[i], shape, std)

    with ThreadPoolExecutor(max_workers=max(1, min(threads, n))) as ex:
        list(ex.map(fill, range(n)))
    return out


@dataclasses.dataclass
class MoEInputs:
    cfg: MoEConfig
    x: np.ndarray              # uint16 bf16 bits [T, d]
    logits: np.ndarray         # float32 [T, E]
    w13: np.ndarray            # uint16 bf16 bits [E, n1, d]
    w2: np.ndarray             # uint16 bf16 bits [E, d, F]
    w13_shared: np.ndarray | None = None   # [n_shared, n1, d]
    w2_shared: np.ndarray | None = None    # [n_shared, d, F]
    router_w: np.ndarray | None = None     # bf16 bits [E, d] (tiny config)


def _logits(cfg: MoEConfig, ss: np.random.SeedSequence, x_bits: np.ndarray):
    rng = np.random.Generator(np.random.PCG64(ss))
    T, E = cfg.T, cfg.E
    router_w = None
    if cfg.logits_kind == "normal":
        lg = rng.standard_normal((T, E)).astype(np.float32)
    elif cfg.logits_kind == "uniform":
        lg = rng.random((T, E), dtype=np.float32)
    elif cfg.logits_kind == "decode_hot":
        # N(0,1) plus a strong bias so that several tokens share experts:
        # +6 on expert 5 for every token and on expert 77 for tokens 0 and 1.
        lg = rng.standard_normal((T, E)).astype(np.float64)
        lg[:, 5 % E] += 6.0
        lg[: min(2, T), 77 % E] += 6.0
        lg = lg.astype(np.float32)
    elif cfg.logits_kind == "zipf":
        # Plackett-Luce sampling of experts with Zipf(1.1) popularity:
        # logit = ln p_rank(e) + Gumbel(0,1); the 8 least popular experts get
        # a -30 bias so that they receive no tokens.
        rank_of = rng.permutation(E)                 # rank (0 = most popular)
        p = (np.arange(1, E + 1, dtype=np.float64)) ** -1.1
        p /= p.sum()
        u = rng.random((T, E))
        gumbel = -np.log(-np.log(np.clip(u, 1e-300, None)))
        lg = np.log(p[rank_of])[None, :] + gumbel
        cold = rank_of >= E - 8
        lg[:, cold] -= 30.0
        lg = lg.astype(np.float32)
    elif cfg.logits_kind == "router":
        # Router projection of the tiny configuration: W_g ~ N(0, 0.02) in
        # bf16, logits = fp32(sum_d x * W_g) accumulated in fp64.  The router
        # GEMM itself is outside the layer's boundary; it only makes inputs.
        router_w = _normal_bf16(ss.spawn(1)[0], (E, cfg.d), 0.02)
        xf = bf16_bits_to_f32(x_bits).astype(np.float64)
        wf = bf16_bits_to_f32(router_w).astype(np.float64)
        lg = (xf @ wf.T).astype(np.float32)
    else:
        raise ValueError(cfg.logits_kind)
    return np.ascontiguousarray(lg, dtype=np.float32), router_w


def make_inputs(cfg: MoEConfig, threads: int = 8) -> MoEInputs:
    """Draw every input of one configuration from its seed."""
    root = np.random.SeedSequence(cfg.seed)
    s_x, s_lg, s_w13, s_w2, s_sh13, s_sh2 = root.spawn(6)
    x = _normal_bf16(s_x, (cfg.T, cfg.d), 1.0)
    logits, router_w = _logits(cfg, s_lg, x)
    w13 = _stack_normal_bf16(s_w13, cfg.E, (cfg.n1, cfg.d), 0.02, threads)
    w2 = _stack_normal_bf16(s_w2, cfg.E, (cfg.d, cfg.F), 0.02, threads)
    w13s = w2s = None
    if cfg.n_shared:
        w13s = _stack_normal_bf16(s_sh13, cfg.n_shared, (cfg.n1, cfg.d), 0.02, threads)
        w2s = _stack_normal_bf16(s_sh2, cfg.n_shared, (cfg.d, cfg.F), 0.02, threads)
    return MoEInputs(cfg, x, logits, w13, w2, w13s, w2s, router_w)


MX_BLOCK = 32     # K values sharing one power-of-two scale
E4M3_MAX = 448.0  # largest finite e4m3 value


def quantize_mxfp8(w_bits: np.ndarray):
    """Weight-only block quantisation of a bf16 stack [E, rows, K] (bits) for
    the fp8 expert weights: every run of 32 consecutive K values of a row
    shares a power-of-two scale 2^s (s the smallest integer with
    max|w| / 2^s <= 448), stored as the byte s + 127; the values w / 2^s are
    rounded to e4m3 (round to nearest even; torch's cast).

    Returns (q uint8 [E, rows, K] e4m3 bit patterns, scales uint8
    [E, K/32, rows]) -- the scales K-block-major, so that the scales of 128
    consecutive rows for one 64-wide K step are two rows of 128 bytes."""
    import torch
    w = bf16_bits_to_f32(w_bits).astype(np.float64)
    E, R, K = w.shape
    assert K % MX_BLOCK == 0
    blocks = w.reshape(E, R, K // MX_BLOCK, MX_BLOCK)
    amax = np.abs(blocks).max(axis=3)
    with np.errstate(divide="ignore"):
        s = np.ceil(np.log2(np.where(amax > 0, amax, 1.0) / E4M3_MAX))
    s = np.clip(s, -126, 127).astype(np.int64)               # byte 1..254
    scaled = blocks / np.exp2(s)[..., None]
    q = torch.from_numpy(scaled.reshape(E, R, K).astype(np.float32)).to(torch.float8_e4m3fn)
    q_bits = q.view(torch.uint8).numpy().copy()
    scales = np.ascontiguousarray((s + 127).astype(np.uint8).transpose(0, 2, 1))
    return q_bits, scales


def fp8_weights(inp: "MoEInputs"):
    """The fp8 form of one configuration's expert weights: (w13_q, w13_s,
    w2_q, w2_s, w13s_q, w13s_s, w2s_q, w2s_s), the shared expert's entries
    None without one."""
    out = list(quantize_mxfp8(inp.w13)) + list(quantize_mxfp8(inp.w2))
    if inp.w13_shared is not None:
        out += list(quantize_mxfp8(inp.w13_shared)) + list(quantize_mxfp8(inp.w2_shared))
    else:
        out += [None] * 4
    return tuple(out)


def grad_output(T: int, d: int, seed: int) -> np.ndarray:
    """Seeded dL/dout for the backward: N(0, 1) in bf16 bits [T, d]."""
    return _normal_bf16(np.random.SeedSequence(seed).spawn(1)[0], (T, d), 1.0)


def router_inputs(T: int, d: int, E: int, seed: int, zero_rows=()):
    """Seeded router-projection inputs: x ~ N(0, 1) and W_g ~ N(0, 0.02),
    both bf16 bits ([T, d] and [E, d]); the listed token rows are zero."""
    ss = np.random.SeedSequence(seed).spawn(2)
    x = _normal_bf16(ss[0], (T, d), 1.0)
    for t in zero_rows:
        x[t] = 0
    return x, _normal_bf16(ss[1], (E, d), 0.02)


def tie_logits(T: int, E: int, seed: int, levels: int = 3) -> np.ndarray:
    """Logits drawn from a handful of values so that ties are everywhere."""
    rng = np.random.Generator(np.random.PCG64(seed))
    vals = np.linspace(-1.0, 1.0, levels).astype(np.float32)
    return np.ascontiguousarray(vals[rng.integers(0, levels, size=(T, E))])


def random_topk_ids(T: int, E: int, k: int, seed: int, skew: float = 0.0) -> np.ndarray:
    """k distinct expert ids per token (optionally skewed towards low ids)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    keys = rng.random((T, E))
    if skew:
        keys = keys * (1.0 + skew * np.arange(E)[None, :])
    return np.ascontiguousarray(np.argsort(keys, axis=1, kind="stable")[:, :k].astype(np.int32))
