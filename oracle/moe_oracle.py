"""CPU fp64 oracle of the fused MoE expert layer.

TEST INFRASTRUCTURE.  Only the test suite, the package smoke check and the
benchmark's CPU-baseline leg may import or run this module.  The product path
(the CUDA library and its Python binding) never calls it, and it shares no
code with that path: no kernels, helpers, tables or pre/post-processing.

Plain, slow and obviously correct: every step is the definition written out,
with numpy sort and matmul as the only library primitives.  Floating point is
fp64 throughout, over the exact fp32 router logits and the exact bf16 values
of activations and weights.  Nothing is rounded to bf16 on the way.

Sources (web pages on fused MoE kernels):

* "Fused MoE Kernel Optimization" (skillmd, zjli2013/fused-moe-kernel):
  section "Token-Expert Routing" (top-k gating, sort by expert, pad each
  expert to a multiple of BLOCK_SIZE_M), "Grouped GEMM Structure"
  (sorted_token_ids, expert_ids, num_tokens_post_padded), "Verification"
  (compare against sequential per-expert matmuls with top-k selection) and
  "Common Pitfalls" (slot // top_k is the token, padding ids are at least
  num_valid_tokens, [E, N, K] weight layout, top-k weights on the right rows).
* axolotl vendor-moe diff, src/axolotl/monkeypatch/deepseek_v3/__init__.py,
  ``_moe_triton_forward``: gate and up projections, ``act_fn(gate) * up``,
  down projection, then the weighted sum over the k expert outputs.
* the same diff, scripts/benchmarks/build_deepseek_v3_8b.py ``build_config``:
  n_group / topk_group grouped routing, norm_topk_prob, routed_scaling_factor
  and one shared expert.
* mlxcel PR "perf(moe): preserve squared-ReLU fused MoE kernel behind a
  dedicated flag", Summary: fc1 -> relu^2 -> fc2 experts with no gate.
* the same axolotl diff, scripts/benchmarks/deepseek_v3_moe.py
  ``timed_forward``: the block's gate maps the flattened hidden states to the
  top-k expert ids and weights (router projection, then gating).
* backward: the same diff's grouped-GEMM backward kernels,
  src/axolotl/kernels/moe/tt_cg_gemm/cg_backward.py (``_kernel_cg_backward_dx``:
  the gradient of the token rows from dY and each expert's weights;
  ``_kernel_cg_backward_dw``: each expert's weight gradient summed over the
  rows routed to it) and the Gemma-4 MoE training note (the expert path of a
  training step, forward and backward), restated as the chain rule.

Readings where the pages are silent (each is also listed in the design notes):

* Selection key is (logit descending, expert index ascending); softmax is
  monotone so selecting on logits selects the same set as on probabilities.
* Group score ``max``: the largest logit of the group.  Group score ``top2``:
  the sum of the two largest logits of the group, rounded to fp32 (one fp32
  addition), so that the group choice, an integer decision, is taken in the
  same precision as the kernel takes it.  Groups are ranked by (score
  descending, group index ascending).
* Renormalised weights: softmax over the k chosen logits.  Otherwise: the
  softmax over all E logits, taken at the chosen experts.  Both are then
  multiplied by routed_scaling.
* Align: slots s = t*k + j are sorted by expert, stably (ascending s); each
  expert's run is padded to a multiple of block_m with the value S = T*k;
  experts with no slot get no block; unused positions also hold S and unused
  block ids hold -1.
* The shared expert is added with weight 1 to every token, unscaled.
"""
from __future__ import annotations

import numpy as np

ACT_SWIGLU = 0
ACT_RELU2 = 1
GROUP_MAX = 0
GROUP_TOP2SUM = 1


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns (uint16) as fp64."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u32.view(np.float32).astype(np.float64)


def e4m3_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of fp8 e4m3 bit patterns (uint8): sign, 4 exponent bits
    (bias 7), 3 mantissa bits; exponent field 0 is subnormal (m * 2^-9);
    S.1111.111 is NaN and there is no infinity (largest value 448)."""
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7).astype(np.float64)
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return sign * val


def dequant_mxfp8(q: np.ndarray, scales: np.ndarray, block: int = 32) -> np.ndarray:
    """fp8 expert weights as fp64: w[.., r, c] = e4m3(q[.., r, c]) *
    2^(scales[.., c // block, r] - 127), with q [..., rows, K] and the scale
    bytes K-block-major [..., K / block, rows]."""
    w = e4m3_to_f64(q)
    s = np.asarray(scales, dtype=np.int64) - 127
    per_col = np.repeat(np.swapaxes(s, -1, -2), block, axis=-1)  # [..., rows, K]
    return w * np.exp2(per_col.astype(np.float64))


# --------------------------------------------------------------------------
# Route
# --------------------------------------------------------------------------

def router_logits(x_bits: np.ndarray, w_gate_bits: np.ndarray) -> np.ndarray:
    """Router projection of the gate: logits[t, e] = sum_i x[t, i] * W_g[e, i]
    over the exact bf16 values, in fp64 (x [T, d], W_g [E, d], bf16 bits)."""
    return bf16_to_f64(x_bits) @ bf16_to_f64(w_gate_bits).T


def _order_desc(values: np.ndarray) -> np.ndarray:
    """Indices ordered by (value descending, index ascending)."""
    # A stable sort of the negated values keeps equal values in index order.
    return np.argsort(-np.asarray(values), kind="stable")


def group_scores(l32: np.ndarray, n_group: int, group_score: int) -> np.ndarray:
    """Score of each contiguous expert group of one token's fp32 logits."""
    E = l32.shape[0]
    g = l32.reshape(n_group, E // n_group)
    if group_score == GROUP_MAX:
        return g.max(axis=1)
    if group_score == GROUP_TOP2SUM:
        srt = np.sort(g, axis=1)[:, ::-1]
        if srt.shape[1] < 2:
            return srt[:, 0].astype(np.float32)
        return (srt[:, 0].astype(np.float32) + srt[:, 1].astype(np.float32)).astype(np.float32)
    raise ValueError("unknown group score")


def route(logits: np.ndarray, k: int, n_group: int = 1, topk_group: int = 1,
          group_score: int = GROUP_MAX, renormalize: bool = True,
          routed_scaling: float = 1.0):
    """Top-k gating over router logits ("Token-Expert Routing", step 1).

    Returns (topk_ids int32 [T,k], topk_weights float64 [T,k]).  ids of a
    token are listed in selection order (logit descending, index ascending).
    """
    logits = np.asarray(logits, dtype=np.float32)
    T, E = logits.shape
    assert E % n_group == 0 and 1 <= topk_group <= n_group
    assert 1 <= k <= (E // n_group) * topk_group
    assert np.isfinite(logits).all(), "non-finite router logits are unsupported"
    ids = np.empty((T, k), dtype=np.int32)
    wts = np.empty((T, k), dtype=np.float64)
    gsize = E // n_group
    for t in range(T):
        l32 = logits[t]
        l = l32.astype(np.float64)
        if n_group > 1:
            gs = group_scores(l32, n_group, group_score)
            keep_groups = _order_desc(gs)[:topk_group]
            allowed = np.zeros(E, dtype=bool)
            for gidx in keep_groups:
                allowed[gidx * gsize:(gidx + 1) * gsize] = True
        else:
            allowed = np.ones(E, dtype=bool)
        cand = np.nonzero(allowed)[0]                 # ascending expert ids
        chosen = cand[_order_desc(l[cand])][:k]
        ids[t] = chosen
        if renormalize:
            m = l[chosen].max()
            e = np.exp(l[chosen] - m)
            w = e / e.sum()
        else:
            m = l.max()
            p = np.exp(l - m)
            w = p[chosen] / p.sum()
        wts[t] = w * float(routed_scaling)
    return ids, wts


# --------------------------------------------------------------------------
# Align
# --------------------------------------------------------------------------

def max_padded(T: int, k: int, E: int, block_m: int) -> int:
    """Worst-case padded length: S + E*(block_m-1), rounded up to block_m."""
    S = T * k
    p = S + E * (block_m - 1)
    return (p + block_m - 1) // block_m * block_m


def align(topk_ids: np.ndarray, E: int, block_m: int):
    """Sort token-slots by expert and pad each expert to block_m.

    "Token-Expert Routing" steps 2-3 and "Grouped GEMM Structure" of the
    fused-moe-kernel page.  Returns (sorted_token_ids [P_max],
    expert_ids [P_max/block_m], num_tokens_post_padded (int),
    inv_pos [S]), all int32 except the count.
    """
    ids2 = np.asarray(topk_ids, dtype=np.int64)
    T, k = ids2.shape
    flat = ids2.reshape(-1)
    S = T * k
    P = max_padded(T, k, E, block_m)
    sorted_ids = np.full(P, S, dtype=np.int32)
    expert_ids = np.full(P // block_m, -1, dtype=np.int32)
    inv_pos = np.full(S, -1, dtype=np.int32)
    pos = 0
    for e in range(E):
        members = np.nonzero(flat == e)[0]        # ascending slot ids
        n = members.size
        if n == 0:
            continue
        nblk = (n + block_m - 1) // block_m
        sorted_ids[pos:pos + n] = members
        inv_pos[members] = pos + np.arange(n)
        expert_ids[pos // block_m: pos // block_m + nblk] = e
        pos += nblk * block_m
    return sorted_ids, expert_ids, pos, inv_pos


# --------------------------------------------------------------------------
# Forward
# --------------------------------------------------------------------------

def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def expert_hidden(x: np.ndarray, w13_e: np.ndarray, act: int) -> np.ndarray:
    """Hidden activation of one expert on rows x [n, d] (fp64).

    SwiGLU: w13_e rows [0, F) are the gate projection, rows [F, 2F) the up
    projection; h = silu(gate) * up.  Squared ReLU: w13_e is fc1 [F, d] and
    h = max(fc1 x, 0)^2.
    """
    return hidden_values(x, bf16_to_f64(w13_e), act)


def hidden_values(x: np.ndarray, W1: np.ndarray, act: int) -> np.ndarray:
    """expert_hidden on an fp64 weight array W1 [n1, d] (any values)."""
    if act == ACT_SWIGLU:
        F = W1.shape[0] // 2
        g = x @ W1[:F].T
        u = x @ W1[F:].T
        return silu(g) * u
    if act == ACT_RELU2:
        a = x @ W1.T
        return np.maximum(a, 0.0) ** 2
    raise ValueError("unknown activation")


def expert_mlp(x: np.ndarray, w13_e: np.ndarray, w2_e: np.ndarray, act: int) -> np.ndarray:
    """One expert on rows x [n, d] (fp64): w2_e [d, F] applied to h."""
    return expert_hidden(x, w13_e, act) @ bf16_to_f64(w2_e).T


def forward(x_bits: np.ndarray, w13: np.ndarray, w2: np.ndarray,
            topk_ids: np.ndarray, topk_weights: np.ndarray, act: int,
            w13_shared: np.ndarray | None = None,
            w2_shared: np.ndarray | None = None) -> np.ndarray:
    """out[t] = sum_j w[t,j] * expert_{ids[t,j]}(x[t])  (+ shared(x[t])).

    Sequential per-expert matmuls with top-k selection ("Verification" of the
    fused-moe-kernel page); returns fp64 [T, d].
    """
    x = bf16_to_f64(x_bits)
    ids = np.asarray(topk_ids)
    wts = np.asarray(topk_weights, dtype=np.float64)
    T, d = x.shape
    out = np.zeros((T, d), dtype=np.float64)
    E = w13.shape[0]
    for e in range(E):
        t_idx, j_idx = np.nonzero(ids == e)
        if t_idx.size == 0:
            continue
        y = expert_mlp(x[t_idx], w13[e], w2[e], act)
        np.add.at(out, t_idx, wts[t_idx, j_idx][:, None] * y)
    if w13_shared is not None:
        for s in range(w13_shared.shape[0]):
            out += expert_mlp(x, w13_shared[s], w2_shared[s], act)
    return out


# --------------------------------------------------------------------------
# Backward
# --------------------------------------------------------------------------
#
# The training pass of the same layer: given dL/dout, the gradients of the
# loss with respect to the tokens, both expert weight stacks and the top-k
# weights.  The pages motivate it by training (the Gemma-4 MoE note: the
# Python-loop expert path dominates a training step; the axolotl diff's
# grouped-GEMM backward kernels compute the gradient of the token rows, dX,
# and of every expert's weights, dW, from the grouped layout).  Here it is
# the chain rule through each expert's MLP, written out per expert over the
# rows routed to it, with no blocking and nothing rounded.


def silu_grad(z: np.ndarray) -> np.ndarray:
    """Derivative of silu(z) = z * sigmoid(z): sigmoid(z) * (1 + z * (1 - sigmoid(z)))."""
    sg = 1.0 / (1.0 + np.exp(-z))
    return sg * (1.0 + z * (1.0 - sg))


def expert_backward_values(x: np.ndarray, W13: np.ndarray, W2: np.ndarray, dy: np.ndarray, act: int):
    """One expert y = W2 act(W13 x) on rows x [n, d], all fp64 arrays, with
    dL/dy = dy [n, d].  Returns (dx [n, d], dW13 [n1, d], dW2 [d, F], y [n, d]).

    SwiGLU: a = [g; u] = W13 x (gate rows first), h = silu(g) * u,
    dh = W2^T dy, dg = dh * u * silu'(g), du = dh * silu(g).
    Squared ReLU: a = W13 x, h = max(a, 0)^2, da = dh * 2 max(a, 0).
    Then dx = W13^T da, dW13 = sum over rows of da x^T, dW2 = sum of dy h^T.
    """
    da, h = expert_backward_hidden(x, W13, W2, dy, act)
    return da @ W13, da.T @ x, dy.T @ h, h @ W2.T


def expert_backward_hidden(x: np.ndarray, W13: np.ndarray, W2: np.ndarray, dy: np.ndarray, act: int):
    """The hidden quantities of expert_backward_values: (da [n, n1], h [n, F])."""
    dh = dy @ W2                                   # [n, F]
    if act == ACT_SWIGLU:
        F = W13.shape[0] // 2
        g = x @ W13[:F].T
        u = x @ W13[F:].T
        h = silu(g) * u
        da = np.concatenate([dh * u * silu_grad(g), dh * silu(g)], axis=1)
    elif act == ACT_RELU2:
        a = x @ W13.T
        h = np.maximum(a, 0.0) ** 2
        da = dh * 2.0 * np.maximum(a, 0.0)
    else:
        raise ValueError("unknown activation")
    return da, h


def backward_values(x: np.ndarray, W13: np.ndarray, W2: np.ndarray, topk_ids: np.ndarray,
                    topk_weights: np.ndarray, act: int, dout: np.ndarray,
                    W13_shared: np.ndarray | None = None, W2_shared: np.ndarray | None = None) -> dict:
    """Gradients of out[t] = sum_j w[t,j] * expert_{ids[t,j]}(x[t]) (+ shared(x[t]))
    for dL/dout = dout, on fp64 arrays: x [T, d], W13 [E, n1, d], W2 [E, d, F].

    Per expert e and the rows (t, j) routed to it: the expert sees dL/dy =
    w[t,j] * dout[t]; dL/dw[t,j] = dout[t] . y_e(x[t]).  Returns a dict with
    dx [T, d], dw13 [E, n1, d], dw2 [E, d, F], dtopk_weights [T, k] and,
    with a shared expert, dw13_shared / dw2_shared [n_shared, ...].
    """
    ids = np.asarray(topk_ids)
    wts = np.asarray(topk_weights, dtype=np.float64)
    T, d = x.shape
    E = W13.shape[0]
    dx = np.zeros((T, d), dtype=np.float64)
    dw13 = np.zeros(W13.shape, dtype=np.float64)
    dw2 = np.zeros(W2.shape, dtype=np.float64)
    dtopk = np.zeros(ids.shape, dtype=np.float64)
    for e in range(E):
        t_idx, j_idx = np.nonzero(ids == e)
        if t_idx.size == 0:
            continue
        w = wts[t_idx, j_idx][:, None]
        gx, gw13, gw2, y = expert_backward_values(x[t_idx], W13[e], W2[e], w * dout[t_idx], act)
        np.add.at(dx, t_idx, gx)
        dw13[e] = gw13
        dw2[e] = gw2
        dtopk[t_idx, j_idx] = np.sum(dout[t_idx] * y, axis=1)
    res = {"dx": dx, "dw13": dw13, "dw2": dw2, "dtopk_weights": dtopk}
    if W13_shared is not None:
        ns = W13_shared.shape[0]
        res["dw13_shared"] = np.zeros(W13_shared.shape, dtype=np.float64)
        res["dw2_shared"] = np.zeros(W2_shared.shape, dtype=np.float64)
        for i in range(ns):
            gx, gw13, gw2, _ = expert_backward_values(x, W13_shared[i], W2_shared[i], dout, act)
            dx += gx
            res["dw13_shared"][i] = gw13
            res["dw2_shared"][i] = gw2
    return res


def backward(x_bits: np.ndarray, w13: np.ndarray, w2: np.ndarray, topk_ids: np.ndarray,
             topk_weights: np.ndarray, act: int, dout_bits: np.ndarray,
             w13_shared: np.ndarray | None = None, w2_shared: np.ndarray | None = None) -> dict:
    """backward_values over the exact values of bf16 inputs (x, weights and
    dL/dout as uint16 bit patterns; topk_weights as given)."""
    return backward_values(bf16_to_f64(x_bits), bf16_to_f64(w13), bf16_to_f64(w2), topk_ids, topk_weights,
                           act, bf16_to_f64(dout_bits),
                           None if w13_shared is None else bf16_to_f64(w13_shared),
                           None if w2_shared is None else bf16_to_f64(w2_shared))


def forward_values(x: np.ndarray, W13: np.ndarray, W2: np.ndarray, topk_ids: np.ndarray,
                   topk_weights: np.ndarray, act: int, W13_shared: np.ndarray | None = None,
                   W2_shared: np.ndarray | None = None) -> np.ndarray:
    """forward on fp64 arrays of any values (x [T, d], W13 [E, n1, d],
    W2 [E, d, F]): sequential per-expert matmuls with top-k selection."""
    ids = np.asarray(topk_ids)
    wts = np.asarray(topk_weights, dtype=np.float64)
    out = np.zeros(x.shape, dtype=np.float64)
    for e in range(W13.shape[0]):
        t_idx, j_idx = np.nonzero(ids == e)
        if t_idx.size == 0:
            continue
        y = hidden_values(x[t_idx], W13[e], act) @ W2[e].T
        np.add.at(out, t_idx, wts[t_idx, j_idx][:, None] * y)
    if W13_shared is not None:
        for i in range(W13_shared.shape[0]):
            out += hidden_values(x, W13_shared[i], act) @ W2_shared[i].T
    return out
