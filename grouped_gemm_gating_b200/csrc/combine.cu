// Weighted scatter-reduce back to token order.
//
// out[t, :] = sum_{j<k} y[inv_pos[t*k + j], :]  (+ y[ntpp + t, :] for the
// shared expert), where each y row already carries its top-k weight (applied
// in the down GEMM epilogue; y is fp32).  This is the final
// `(expert_outputs * topk_weights).sum(dim=1)` of the axolotl
// `_moe_triton_forward` (src/axolotl/monkeypatch/deepseek_v3/__init__.py)
// and "Common Pitfalls" 4 of the fused-moe-kernel page (weights on the right
// rows).  The sum is fp32 in slot order, so the result is deterministic.
//
// HBM-bound: each thread moves 8 columns (two 16-byte fp32 vectors in per
// row, one 16-byte bf16 vector out); one block per token row, columns
// strided over the block.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kCombineThreads = 256;

__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const float* __restrict__ y, const int32_t* __restrict__ inv_pos,
                   const int32_t* __restrict__ ntpp, int T, int k, int d, int has_shared,
                   uint16_t* __restrict__ out) {
  const int t = blockIdx.x;
  pdl_wait();
  pdl_launch_dependents();
  if (t >= T) return;
  const int nvec = d / 8;
  int rows[MOE_MAX_TOPK + 1];
  int nrows = 0;
  for (int j = 0; j < k; ++j) rows[nrows++] = inv_pos[static_cast<size_t>(t) * k + j];
  if (has_shared) rows[nrows++] = *ntpp + t;
  for (int v = threadIdx.x; v < nvec; v += kCombineThreads) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    for (int r = 0; r < nrows; ++r) {
      const float4* src = reinterpret_cast<const float4*>(y + static_cast<size_t>(rows[r]) * d + v * 8);
      const float4 a = src[0], b = src[1];
      acc[0] += a.x;
      acc[1] += a.y;
      acc[2] += a.z;
      acc[3] += a.w;
      acc[4] += b.x;
      acc[5] += b.y;
      acc[6] += b.z;
      acc[7] += b.w;
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * d + v * 8) = o;
  }
}

}  // namespace

cudaError_t launch_combine(const float* y, const int32_t* inv_pos, const int32_t* ntpp, int T, int k, int d,
                           int has_shared, uint16_t* out, cudaStream_t stream, int* launches) {
  ++*launches;
  return launch_pdl(combine_kernel, dim3(T), dim3(kCombineThreads), 0, stream, y, inv_pos, ntpp, T, k, d, has_shared,
                    out);
}

}  // namespace moe
