/*
 * moe.h — C ABI of the B200 (sm_100a) fused Mixture-of-Experts expert layer.
 *
 * The layer computes, for T tokens x[T, d] and router logits[T, E]:
 *
 *   1. moe_route   top-k gating: per token, the k experts with the largest
 *                  logits (optionally restricted to the topk_group best of
 *                  n_group contiguous expert groups) and their softmax
 *                  weights (renormalised over the chosen k, or the full
 *                  softmax), times routed_scaling.
 *   2. moe_align   the token-slots s = t*k + j sorted by expert (stable in
 *                  s), each expert's run padded to a multiple of block_m:
 *                  sorted_token_ids, expert_ids (one per block of block_m
 *                  rows), num_tokens_post_padded and the inverse map inv_pos.
 *   3. moe_forward the grouped gate/up GEMM over [E, N, K] expert weights
 *                  with a fused SwiGLU or squared-ReLU epilogue, the grouped
 *                  down GEMM with the top-k weight applied per row, and the
 *                  weighted scatter-reduce back to out[T, d] (plus an
 *                  optional always-on shared expert).
 *
 * Sources.  "Fused MoE Kernel Optimization" (skillmd zjli2013/fused-moe-
 * kernel): "Token-Expert Routing" (top-k gating; sort tokens by expert; pad
 * each expert's count to a multiple of BLOCK_SIZE_M), "Grouped GEMM
 * Structure" (sorted_token_ids maps blocks to token rows, expert_ids maps
 * each M-block to its expert, blocks at or past num_tokens_post_padded do no
 * work) and "Common Pitfalls" (slot // top_k is the token; padding ids are at
 * least num_valid_tokens; [E, N, K] expert-major weights; top-k weights on
 * the right rows).  The axolotl vendor-moe diff,
 * src/axolotl/monkeypatch/deepseek_v3/__init__.py `_moe_triton_forward`
 * (gate/up GEMMs, act_fn(gate) * up, down GEMM, weighted sum over k) and
 * scripts/benchmarks/build_deepseek_v3_8b.py `build_config` (n_group,
 * topk_group, routed_scaling_factor, norm_topk_prob, one shared expert).
 * The mlxcel PR "perf(moe): preserve squared-ReLU fused MoE kernel behind a
 * dedicated flag", Summary (fc1 -> relu^2 -> fc2 experts with no gate).
 *
 * Conventions for every call.
 *   - Pointers named `dev`/tensors are DEVICE pointers (cudaMalloc'd or
 *     torch-owned), row-major, contiguous and 16-byte aligned.  The caller
 *     owns every buffer; the library allocates nothing and keeps no state
 *     between calls apart from one-time per-device kernel attribute set-up.
 *   - bf16 values are passed as raw 16-bit patterns (uint16_t).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and never synchronise the host; device-side results
 *     such as num_tokens_post_padded stay on the device.
 *   - Every argument is checked on the host first.  A failed check returns
 *     an error code and launches nothing.  T == 0 is MOE_OK and a no-op
 *     (moe_align still writes its padding outputs).
 *   - `dev_status` (nullable) is one int32 on the device.  Kernels that
 *     detect an error at run time (non-finite logits, an out-of-range expert
 *     id, a pipeline wait that exceeded its time limit) store the first such
 *     code there with an atomic compare-and-swap; they never trap.  Clear it
 *     to 0 before use; read it with moe_read_status.
 */
#ifndef MOE_B200_H_
#define MOE_B200_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* identical to cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,    /* shape, pointer, alignment or range check failed */
  MOE_ERR_UNSUPPORTED = 2,    /* valid arguments outside the library's limits */
  MOE_ERR_WORKSPACE = 3,      /* workspace pointer missing or too small */
  MOE_ERR_CUDA = 4,           /* a CUDA runtime/driver call failed (launch, attribute, tensor map) */
  MOE_ERR_NONFINITE = 5,      /* device: a router logit was NaN or infinite */
  MOE_ERR_DEVICE_TIMEOUT = 6, /* device: a pipeline wait exceeded its time limit; outputs are invalid */
  MOE_ERR_BAD_EXPERT_ID = 7   /* device: a topk_ids entry was outside [0, E) */
} moe_status;

typedef enum { MOE_ACT_SWIGLU = 0, MOE_ACT_RELU2 = 1 } moe_act;

typedef enum {
  MOE_GROUP_MAX = 0,     /* group score = largest logit in the group */
  MOE_GROUP_TOP2SUM = 1  /* group score = fp32 sum of the two largest logits in the group */
} moe_group_score;

/* Limits of the library (checked; MOE_ERR_UNSUPPORTED beyond them):
 *   1 <= E <= 256, 1 <= k <= min(E, 16), d and F multiples of 64 with
 *   64 <= d, F <= 16384, block_m in {16, 32, 64, 128}, n_shared in {0, 1},
 *   T * k < 2^30. */
#define MOE_MAX_EXPERTS 256
#define MOE_MAX_TOPK 16

/* Worst-case padded length of sorted_token_ids for (T, k, E, block_m):
 * P_max = T*k + E*(block_m - 1), rounded up to a multiple of block_m.
 * Returns -1 on invalid arguments. */
MOE_API int64_t moe_max_padded(int T, int k, int E, int block_m);

/* Bytes of device scratch moe_align needs (0 when T*k is small enough for
 * the single-block path).  Returns 0 on invalid arguments. */
MOE_API size_t moe_align_workspace_size(int T, int k, int E);

/* Bytes of device scratch moe_forward needs: a 64 KiB block of int32
 * counters, then (block_m = 128 only) the activation h [P_total, F] in bf16,
 * then the fp32 output accumulator [T, d], then (block_m = 128, d >= 1024 and
 * F >= 1024) the token rows in expert-sorted order [P_total, d] in bf16, where
 * P_total = P_max + n_shared * ceil(T / block_m) * block_m.
 * The counter block (the first 64 KiB after rounding ws up to 256 bytes)
 * must be zero before the first moe_forward on a workspace (allocate it
 * zero-filled or cudaMemset it once).  The kernels keep it consistent from
 * one call to the next -- also after a call whose kernel gave up on a wait
 * (MOE_ERR_DEVICE_TIMEOUT): every CTA counts itself out on every exit path,
 * the last one returns the two grid counters to zero, and the third word is
 * a release generation that only moves forward -- so a workspace can be
 * reused across calls and layer shapes, errors included, as long as nothing
 * else writes that block.  Returns 0 on invalid arguments. */
MOE_API size_t moe_workspace_size(int T, int d, int F, int E, int k, int block_m,
                          moe_act act, int n_shared);

/*
 * moe_route — top-k gating ("Token-Expert Routing", step 1).
 *   logits        [T, E] fp32, device.
 *   n_group       number of contiguous expert groups (1 = ungrouped); E % n_group == 0.
 *   topk_group    groups kept per token, 1 <= topk_group <= n_group;
 *                 k <= topk_group * E / n_group.
 *   group_score   how a group is scored (ignored when n_group == 1).
 *   renormalize   1: softmax over the k chosen logits; 0: full softmax over E.
 *   routed_scaling multiplies every weight (finite, > 0).
 *   topk_ids      [T, k] int32 out, device: ids in selection order (logit
 *                 descending, ties to the lower expert id).
 *   topk_weights  [T, k] fp32 out, device.
 * Groups are ranked by (score descending, group index ascending).  Errors:
 * MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED on the host; MOE_ERR_NONFINITE
 * in dev_status if a logit is NaN/Inf (outputs then unspecified).
 */
MOE_API moe_status moe_route(const float* logits, int T, int E, int k,
                     int n_group, int topk_group, moe_group_score group_score,
                     int renormalize, float routed_scaling,
                     int32_t* topk_ids, float* topk_weights,
                     int32_t* dev_status, moe_stream_t stream);

/*
 * moe_router — the gate of the MoE block in one call: router projection
 * logits = x . W_g^T (W_g [E, d_model]) and top-k gating.  In the axolotl
 * DeepSeek-V3 benchmark (scripts/benchmarks/deepseek_v3_moe.py,
 * timed_forward) the block's gate maps the flattened hidden states to their
 * top-k expert ids and weights; "Fused MoE Kernel Optimization" (overview:
 * top-k gating fusion; "Token-Expert Routing" step 1) gates on those
 * logits.  Here the product runs on the tensor cores (or, for small
 * batches, the CUDA cores) and a warp per token gates the logits.
 *   x             [T, d] bf16, device, row-major; d a multiple of 64.
 *   w_gate        [E, d] bf16, device, row-major (K = d contiguous); E <= 256.
 *   k, n_group, topk_group, group_score, renormalize, routed_scaling:
 *                 as for moe_route; k <= 16.
 *   logits        [T, E] fp32 out, device (4-byte aligned): x . W_g^T with
 *                 fp32 accumulation of the exact bf16 products.
 *   topk_ids, topk_weights: [T, k] out, device: the same values moe_route
 *                 writes for these logits (ids bit for bit, weights up to
 *                 the rounding of the softmax sum).
 * Up to 1024 tokens (and d <= 5120) the product runs on the CUDA cores, in
 * CTAs of 8 expert rows x 16 tokens; larger batches run on the tensor cores
 * (128-token tiles, W_g's rows as the N = 256 operand).  Either way the
 * routing kernel then gates the written logits (two launches).  T == 0 is a
 * no-op.
 * Errors as for moe_route; x and w_gate must be 16-byte aligned.
 */
MOE_API moe_status moe_router(const uint16_t* x, int T, int d, const uint16_t* w_gate, int E, int k,
                     int n_group, int topk_group, moe_group_score group_score,
                     int renormalize, float routed_scaling,
                     float* logits, int32_t* topk_ids, float* topk_weights,
                     int32_t* dev_status, moe_stream_t stream);

/*
 * moe_align — sort token-slots by expert and pad to block_m ("Token-Expert
 * Routing" steps 2-3, "Grouped GEMM Structure", "Common Pitfalls" 1-2).
 *   topk_ids               [T, k] int32, device, values in [0, E).
 *   sorted_token_ids       [P_max] int32 out: slot ids s = t*k + j grouped by
 *                          expert (ascending expert, ascending s within an
 *                          expert); every other entry holds S = T*k.
 *   expert_ids             [P_max / block_m] int32 out: the expert of each
 *                          block; -1 for blocks at or past the padded total.
 *   num_tokens_post_padded [1] int32 out: sum_e ceil(count_e/block_m)*block_m.
 *   inv_pos                [T*k] int32 out: position of slot s in sorted_token_ids.
 *   ws, ws_bytes           scratch of moe_align_workspace_size bytes (may be
 *                          NULL when that size is 0).
 * Experts with no slot get no block.  Results are unique and deterministic.
 * An id outside [0, E) sets MOE_ERR_BAD_EXPERT_ID in dev_status.
 */
MOE_API moe_status moe_align(const int32_t* topk_ids, int T, int k, int E, int block_m,
                     int32_t* sorted_token_ids, int32_t* expert_ids,
                     int32_t* num_tokens_post_padded, int32_t* inv_pos,
                     void* ws, size_t ws_bytes,
                     int32_t* dev_status, moe_stream_t stream);

/*
 * moe_forward — grouped expert GEMMs and weighted scatter-reduce.
 *   x            [T, d] bf16.
 *   w13          SwiGLU: [E, 2F, d] bf16, rows [0, F) the gate projection,
 *                rows [F, 2F) the up projection.  relu^2: [E, F, d] (fc1).
 *   w2           [E, d, F] bf16 (down projection / fc2).
 *   w13_shared, w2_shared  the shared expert, same layouts with E = 1
 *                (required iff n_shared == 1).
 *   topk_weights [T, k] fp32; sorted_token_ids, expert_ids,
 *                num_tokens_post_padded, inv_pos: moe_align's outputs for
 *                the same (T, k, E, block_m).
 *   out          [T, d] bf16 out:
 *                out[t] = sum_j topk_weights[t,j] * W2_e (act(W13_e x[t]))
 *                         (+ shared(x[t]) with weight 1),
 *                with fp32 accumulation; h is rounded to bf16 (it feeds the
 *                bf16 down GEMM) and the weighted sum is fp32, rounded once
 *                to bf16.  The per-slot (block_m = 128) or per-h-slice
 *                (block_m <= 64) partial results are added into the fp32
 *                accumulator with atomics, in an order that depends on
 *                timing, so repeated calls agree up to the fp32 rounding
 *                of that sum (one bf16 ulp of a result, a little more where
 *                the k terms cancel).  Callers that need bit-identical
 *                outputs from run to run (a training run replayed for
 *                debugging, golden-output regression checks) do not get
 *                them from this call; routing, align and (moe_backward)
 *                the weight gradients are deterministic.  inv_pos is
 *                accepted for interface stability and not read (it may be
 *                NULL).
 *   ws, ws_bytes scratch of moe_workspace_size bytes (its counter block zero
 *                before the first call, see moe_workspace_size); calls sharing
 *                a workspace must not overlap on the GPU.
 * Errors: host checks as above; MOE_ERR_DEVICE_TIMEOUT in dev_status if a
 * pipeline wait inside a GEMM kernel exceeded its limit (out is then invalid;
 * the workspace stays usable for the next call).
 */
MOE_API moe_status moe_forward(const uint16_t* x, int T, int d,
                       const uint16_t* w13, const uint16_t* w2, int E, int F,
                       const uint16_t* w13_shared, const uint16_t* w2_shared, int n_shared,
                       const float* topk_weights, int k,
                       const int32_t* sorted_token_ids, const int32_t* expert_ids,
                       const int32_t* num_tokens_post_padded, const int32_t* inv_pos,
                       int block_m, moe_act act,
                       uint16_t* out, void* ws, size_t ws_bytes,
                       int32_t* dev_status, moe_stream_t stream);

/*
 * moe_forward_fp8 / moe_layer_fp8 -- moe_forward / moe_layer with the
 * expert weights quantised to fp8, for the bandwidth-bound small-batch
 * shapes.  The decode stacks on the pages run MoE experts from quantised
 * weights (the B70 lab page's Q8_0 "Grouped Reordered-Q8" expert path,
 * Intent; the mlxcel PR's quantised `gather_qmm` experts, Summary); here
 * the format is weight-only MXFP8: e4m3 values, and for every run of 32
 * consecutive K values of a weight row one power-of-two scale 2^(b - 127)
 * stored as the byte b (1 <= b <= 254).  The kernel streams the fp8 bytes
 * (halving the weight bytes of the bf16 layer) and expands them in shared
 * memory to bf16 -- exactly: an e4m3 value times a power of two has at most
 * 4 significant bits -- before the same bf16 tensor-core MMAs, so the result
 * is the bf16 layer's on the dequantised weights.
 *   w13_q       [E, N1, d] uint8 e4m3 (layout of moe_forward's w13).
 *   w13_scales  [E, d / 32, N1] uint8 (K-block-major: the scales of one
 *               32-wide block of K for all N1 rows are contiguous).
 *   w2_q        [E, d, F] uint8 e4m3; w2_scales [E, F / 32, d] uint8.
 *   w13s_* / w2s_*  the shared expert, same layouts with E = 1 (n_shared == 1).
 * Everything else as for moe_forward / moe_layer.  block_m must be 16, 32 or
 * 64 (the fused expert kernel; MOE_ERR_UNSUPPORTED otherwise).  All weight
 * and scale pointers 16-byte aligned.
 */
MOE_API moe_status moe_forward_fp8(const uint16_t* x, int T, int d,
                           const uint8_t* w13_q, const uint8_t* w13_scales,
                           const uint8_t* w2_q, const uint8_t* w2_scales, int E, int F,
                           const uint8_t* w13s_q, const uint8_t* w13s_scales,
                           const uint8_t* w2s_q, const uint8_t* w2s_scales, int n_shared,
                           const float* topk_weights, int k,
                           const int32_t* sorted_token_ids, const int32_t* expert_ids,
                           const int32_t* num_tokens_post_padded, const int32_t* inv_pos,
                           int block_m, moe_act act,
                           uint16_t* out, void* ws, size_t ws_bytes,
                           int32_t* dev_status, moe_stream_t stream);

MOE_API moe_status moe_layer_fp8(const float* logits, int T, int E, int k,
                         int n_group, int topk_group, moe_group_score group_score,
                         int renormalize, float routed_scaling,
                         const uint16_t* x, int d,
                         const uint8_t* w13_q, const uint8_t* w13_scales,
                         const uint8_t* w2_q, const uint8_t* w2_scales, int F,
                         const uint8_t* w13s_q, const uint8_t* w13s_scales,
                         const uint8_t* w2s_q, const uint8_t* w2s_scales, int n_shared,
                         int block_m, moe_act act,
                         int32_t* topk_ids, float* topk_weights,
                         int32_t* sorted_token_ids, int32_t* expert_ids,
                         int32_t* num_tokens_post_padded, int32_t* inv_pos,
                         uint16_t* out, void* ws, size_t ws_bytes,
                         int32_t* dev_status, moe_stream_t stream);

/*
 * moe_align_noalloc — moe_align for callers that cannot allocate device
 * memory.  No passage of the source pages has a counterpart: it is the same
 * sort and pad as moe_align, with the same arguments minus the workspace.
 * Callers that cannot call cudaMalloc (a runtime that reserves all device
 * memory up front, code running while a stream is captured into a CUDA
 * graph, a plugin whose host framework owns every allocation) cannot supply
 * moe_align's workspace; this entry point keeps the multi-block path's
 * scratch in a fixed 1 MiB static device array instead.
 *   Limit: ceil(T*k / 2048) * E <= 262144 (e.g. T*k <= 2^22 at E = 128);
 *   larger problems return MOE_ERR_UNSUPPORTED and launch nothing.
 *   Every GPU that loads the library holds the 1 MiB until the process exits.
 *   The first call on a device looks up the array's device address (one
 *   cudaGetSymbolAddress, cached per device together with its context, and
 *   looked up again when the device's context changes, e.g. after
 *   cudaDeviceReset); make that first call, and the first after such a
 *   change, before any stream capture.  It allocates nothing, ever.
 *   All calls share the one array and it keeps the last call's contents
 *   (nothing in it needs to start at zero); calls whose kernels overlap on
 *   the GPU (other streams, other host threads) race on it and must be
 *   serialised by the caller.
 */
MOE_API moe_status moe_align_noalloc(const int32_t* topk_ids, int T, int k, int E, int block_m,
                             int32_t* sorted_token_ids, int32_t* expert_ids,
                             int32_t* num_tokens_post_padded, int32_t* inv_pos,
                             int32_t* dev_status, moe_stream_t stream);

/*
 * moe_route_align — moe_route followed by moe_align, in one call.  Same
 * arguments, outputs and errors as the two calls; the results are
 * bit-identical.  For small batches (T <= 64, T*k <= 1024, n_group <= 64)
 * both steps run in a single one-block kernel, which saves a launch on the
 * latency-bound decode path; otherwise the two kernels of the separate calls
 * run back to back.  ws / ws_bytes as for moe_align.
 */
MOE_API moe_status moe_route_align(const float* logits, int T, int E, int k,
                           int n_group, int topk_group, moe_group_score group_score,
                           int renormalize, float routed_scaling, int block_m,
                           int32_t* topk_ids, float* topk_weights,
                           int32_t* sorted_token_ids, int32_t* expert_ids,
                           int32_t* num_tokens_post_padded, int32_t* inv_pos,
                           void* ws, size_t ws_bytes,
                           int32_t* dev_status, moe_stream_t stream);

/*
 * moe_layer — the whole layer in one call: moe_route, moe_align and
 * moe_forward on the same arguments, with the same outputs (topk_ids,
 * topk_weights, sorted_token_ids, expert_ids, num_tokens_post_padded and
 * inv_pos are written as by moe_route_align; out as by moe_forward) and the
 * same errors.  No passage of the source pages has this entry point: it is
 * the three calls of "Token-Expert Routing" and "Grouped GEMM Structure"
 * chained, for callers that hold only the router logits.  With block_m = 16,
 * T*k <= 256 and n_group <= 64 (decode / verifier batches) it is one kernel
 * launch: every CTA of the fused expert kernel routes and sorts all tokens
 * in shared memory before streaming weights, and one CTA also writes the
 * routing and align outputs.  Otherwise the routing / align kernels and the
 * forward kernels run back to back.
 *   ws, ws_bytes  scratch of moe_workspace_size(T, d, F, E, k, block_m, act,
 *                 n_shared) bytes (its counter block zero, as for
 *                 moe_forward); the align scratch, when one is needed, is
 *                 carved from it.
 */
MOE_API moe_status moe_layer(const float* logits, int T, int E, int k,
                     int n_group, int topk_group, moe_group_score group_score,
                     int renormalize, float routed_scaling,
                     const uint16_t* x, int d, const uint16_t* w13, const uint16_t* w2, int F,
                     const uint16_t* w13_shared, const uint16_t* w2_shared, int n_shared,
                     int block_m, moe_act act,
                     int32_t* topk_ids, float* topk_weights,
                     int32_t* sorted_token_ids, int32_t* expert_ids,
                     int32_t* num_tokens_post_padded, int32_t* inv_pos,
                     uint16_t* out, void* ws, size_t ws_bytes,
                     int32_t* dev_status, moe_stream_t stream);

/* Bytes of device scratch moe_backward needs: the token rows and the dL/dout
 * rows in expert-sorted order [P_total, d] bf16 each, the gate/up
 * pre-activations [P_total, n1] fp32, their gradient [P_total, n1] bf16,
 * w * h [P_total, F] bf16 and the fp32 dx accumulator [T, d], each 256-byte
 * aligned, where P_total is that of moe_workspace_size with block_m = 128
 * and n1 = 2F (SwiGLU) or F (relu^2).  Returns 0 on invalid arguments. */
MOE_API size_t moe_backward_workspace_size(int T, int d, int F, int E, int k, moe_act act, int n_shared);

/*
 * moe_backward -- the layer's training pass: given dL/dout, the gradients of
 * the loss with respect to the tokens, both expert weight stacks and the
 * top-k weights.  The computation is the grouped backward of the axolotl
 * vendor-moe diff (src/axolotl/kernels/moe/tt_cg_gemm/cg_backward.py:
 * `_kernel_cg_backward_dx`, the token rows' gradient from dY and each
 * expert's weights; `_kernel_cg_backward_dw`, each expert's weight gradient
 * summed over the rows routed to it), for the training use case of the
 * Gemma-4 MoE note (the expert path of a training step).  With, per routed
 * row (t, j) of expert e and its weight w = topk_weights[t, j]:
 *   SwiGLU: [g; u] = W13_e x[t], h = silu(g) u, dh = w W2_e^T dout[t],
 *           da = [dh u silu'(g); dh silu(g)];  relu^2: a = W13_e x[t],
 *           h = max(a, 0)^2, da = 2 dh max(a, 0);
 *   dx[t]        = sum_j W13_e^T da            (+ the shared expert's, w = 1)
 *   dw13[e]      = sum over e's rows of da x[t]^T
 *   dw2[e]       = sum over e's rows of w dout[t] h^T
 *   dtopk[t, j]  = dout[t] . W2_e h
 * Arguments as for moe_forward, with moe_align's outputs for block_m = 128
 * (sorted_token_ids, expert_ids, num_tokens_post_padded; no other block
 * size), plus:
 *   dout          [T, d] bf16, device: dL/dout.
 *   dx            [T, d] bf16 out.
 *   dw13, dw2     [E, n1, d] and [E, d, F] bf16 out (experts no token was
 *                 routed to get zeros); dw13_shared / dw2_shared [1, n1, d] /
 *                 [1, d, F] with n_shared == 1.
 *   dtopk_weights [T, k] fp32 out, nullable (16-byte aligned).
 *   ws, ws_bytes  scratch of moe_backward_workspace_size bytes (no
 *                 initial contents needed).
 * Precision: fp32 accumulation; the recomputed pre-activations stay fp32;
 * da and w*h are rounded to bf16 (the bf16 operands of the next GEMMs); dx is
 * summed over its k rows in fp32 with atomics (in a timing-dependent order)
 * and rounded once; each dW is one fp32 accumulation rounded once.
 * Launches: two row copies, four tcgen05 GEMMs, a conversion and two
 * per-expert weight-gradient GEMMs, all on `stream`.  Errors as for
 * moe_forward.
 */
MOE_API moe_status moe_backward(const uint16_t* x, int T, int d,
                        const uint16_t* w13, const uint16_t* w2, int E, int F,
                        const uint16_t* w13_shared, const uint16_t* w2_shared, int n_shared,
                        const float* topk_weights, int k,
                        const int32_t* sorted_token_ids, const int32_t* expert_ids,
                        const int32_t* num_tokens_post_padded, moe_act act,
                        const uint16_t* dout, uint16_t* dx, uint16_t* dw13, uint16_t* dw2,
                        uint16_t* dw13_shared, uint16_t* dw2_shared, float* dtopk_weights,
                        void* ws, size_t ws_bytes, int32_t* dev_status, moe_stream_t stream);

/* Synchronises `stream`, then returns the code stored in dev_status (MOE_OK
 * when 0), or MOE_ERR_CUDA if the synchronisation or the copy failed. */
MOE_API moe_status moe_read_status(const int32_t* dev_status, moe_stream_t stream);

/* Static, human-readable name of a status code. */
MOE_API const char* moe_status_string(moe_status status);

/* Number of kernel launches the most recent successful call on this host
 * thread issued (for launch accounting in benchmarks). */
MOE_API int moe_last_launch_count(void);

/*
 * moe_debug_timeouts -- test hook for the bounded waits; not for production.
 * No passage of the source pages has a counterpart: it exists so that tests
 * can drive the error path of the kernels' pipeline waits without faulting
 * or hanging the GPU.  Every wait inside the library's kernels (mbarrier
 * phases, grid counters) gives up after a time limit, records
 * MOE_ERR_DEVICE_TIMEOUT in dev_status, waits for its own TMA loads and MMAs
 * still in flight, frees its tensor memory and returns.
 *   wait_limit_ns         limit for kernels launched afterwards, from any
 *                         host thread (0 restores the default of 2 s).
 *   unreachable_arrivals  > 0: kernels launched afterwards wait for that many
 *                         more arrivals than ever come, so the wait runs out
 *                         after the limit: the fused expert kernel (block_m
 *                         <= 64) at its start barrier (more CTAs than its
 *                         grid has), the grouped GEMM kernels (block_m = 128,
 *                         the router's tensor-core path) at their first
 *                         accumulator-full barrier (more commits than the
 *                         MMA issuer makes); 0 restores normal launches.
 * Process-wide; calls that overlap a launch in another thread race with it.
 * MOE_ERR_INVALID_ARG for unreachable_arrivals outside [0, 1024].
 */
MOE_API moe_status moe_debug_timeouts(uint64_t wait_limit_ns, int unreachable_arrivals);

/* Stage profiling (host-thread local).  While enabled, every moe_route,
 * moe_align and moe_forward call records a pair of CUDA events on its stream
 * around each of its kernels (events come from a pool the library owns; the
 * calls may be captured into a CUDA graph, where the records become event
 * nodes that are re-recorded at every replay).
 * Stages: 0 route, 1 align, 2 gate/up (fc1) GEMM, 3 down GEMM, 4 combine
 * (the accumulator's conversion to bf16), 5 fused route+align
 * (moe_route_align on a small batch), 6 fused expert kernel (moe_forward
 * with block_m <= 64: both GEMMs and the scatter-reduce; under moe_layer on
 * a small batch also the routing and align), 7 permute (x rows copied into
 * the expert-sorted order for the gate/up GEMM on CTA pairs, and the
 * backward's row copies), 8 router (moe_router), and for moe_backward: 9
 * pre-activation recompute, 10 dh GEMM with the activation's derivative,
 * 11 dx GEMM, 12 dW13 GEMM, 13 dW2 GEMM (its conversion of dx is stage 4).
 * moe_profile_enable(1) starts a fresh record (and primes the event pool),
 * (0) stops recording and keeps what was recorded.  moe_profile_collect waits for the recorded events,
 * writes into stage_ms[i] (i < n_stages) the summed milliseconds of stage i
 * and into stage_calls[i] (nullable) how many launches were summed; with
 * release != 0 it then returns the events to the pool and clears the record
 * (release == 0 keeps them, e.g. to read a graph's events after each
 * replay).  MOE_ERR_CUDA if an event call failed. */
#define MOE_NUM_STAGES 14
MOE_API moe_status moe_profile_enable(int on);
MOE_API moe_status moe_profile_collect(double* stage_ms, int* stage_calls, int n_stages, int release);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H_ */
