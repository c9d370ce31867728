// Router projection for small and mid-size token batches: logits[t, e] =
// x[t] . W_g[e] on the CUDA cores.  The gate of the MoE block (axolotl DeepSeek-V3
// benchmark, scripts/benchmarks/deepseek_v3_moe.py, timed_forward: the gate
// maps the flattened hidden states to their top-k experts) starts with this
// product; with a handful of tokens it is a matrix-vector product bound by
// reading W_g once, which one tensor-core tile per 128 tokens would stream
// through a single SM.  Here a CTA takes 8 experts x 16 tokens: every warp
// owns one expert row of W_g (16-byte loads, one pass; the other token
// chunks read it from L2) and the CTA's tokens sit in shared memory; products of the
// bf16 values are exact in fp32 and summed in fp32 (per-lane partial sums,
// then a warp tree), within the same d * 2^-24 * sum|x w| bound as the
// tensor-core path.  The top-k gating then runs in the routing kernel.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kGemvWarps = 8;  // experts per CTA

__global__ void __launch_bounds__(kGemvWarps * 32)
    router_gemv_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ w_gate, int T_all, int d, int E,
                       float* __restrict__ logits) {
  extern __shared__ __align__(16) uint16_t xs[];  // [chunk tokens][d]
  pdl_wait();
  pdl_launch_dependents();
  // this CTA's token chunk: rows t0 .. t0 + T - 1
  const int t0 = blockIdx.y * kRouterGemvMaxT;
  const int T = min(kRouterGemvMaxT, T_all - t0);
  x += static_cast<size_t>(t0) * d;
  logits += static_cast<size_t>(t0) * E;
  // stage the tokens (T * d bf16, 16 bytes per thread per step)
  const int n16 = T * d / 8;
  for (int i = threadIdx.x; i < n16; i += blockDim.x)
    reinterpret_cast<uint4*>(xs)[i] = __ldg(reinterpret_cast<const uint4*>(x) + i);
  __syncthreads();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int e = blockIdx.x * kGemvWarps + warp;
  if (e >= E) return;
  const uint4* wrow = reinterpret_cast<const uint4*>(w_gate + static_cast<size_t>(e) * d);
  float acc[kRouterGemvMaxT];
#pragma unroll
  for (int t = 0; t < kRouterGemvMaxT; ++t) acc[t] = 0.0f;
  for (int c = lane; c < d / 8; c += 32) {
    const uint4 wv = __ldg(wrow + c);
    const uint32_t wp[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int t = 0; t < kRouterGemvMaxT; ++t) {
      if (t < T) {
        const uint4 xv = reinterpret_cast<const uint4*>(xs + static_cast<size_t>(t) * d)[c];
        const uint32_t xp[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[t] = fmaf(bf16_bits_to_float(static_cast<uint16_t>(wp[q] & 0xFFFFu)),
                        bf16_bits_to_float(static_cast<uint16_t>(xp[q] & 0xFFFFu)), acc[t]);
          acc[t] = fmaf(bf16_bits_to_float(static_cast<uint16_t>(wp[q] >> 16)),
                        bf16_bits_to_float(static_cast<uint16_t>(xp[q] >> 16)), acc[t]);
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < kRouterGemvMaxT; ++t) {
    if (t < T) {
      float v = acc[t];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == 0) logits[static_cast<size_t>(t) * E + e] = v;
    }
  }
}

}  // namespace

cudaError_t launch_router_gemv(const uint16_t* x, const uint16_t* w_gate, int T, int d, int E, float* logits,
                               cudaStream_t stream, int* launches) {
  if (T < 1 || d % 8 != 0) return cudaErrorInvalidValue;
  const int chunk = T < kRouterGemvMaxT ? T : kRouterGemvMaxT;
  const size_t smem = static_cast<size_t>(chunk) * d * 2;
  if (smem > 48 * 1024) {
    cudaError_t err = cudaFuncSetAttribute(router_gemv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
  }
  const dim3 grid((E + kGemvWarps - 1) / kGemvWarps, (T + kRouterGemvMaxT - 1) / kRouterGemvMaxT);
  cudaError_t err = launch_pdl(router_gemv_kernel, grid, dim3(kGemvWarps * 32), smem, stream, x, w_gate, T, d, E,
                               logits);
  if (err == cudaSuccess && launches) ++*launches;
  return err;
}

}  // namespace moe
