// Last step of the weighted scatter-reduce for token-major tiles: the down
// GEMM has already added every slot's top-k-weighted output (and the shared
// expert's, weight 1) into an fp32 [T, d] accumulator at its token's row --
// the `(expert_outputs * topk_weights).sum(dim=1)` of the axolotl
// `_moe_triton_forward` (src/axolotl/monkeypatch/deepseek_v3/__init__.py),
// "Common Pitfalls" 4 of the fused-moe-kernel page -- so what is left is one
// rounding of each sum to bf16.
//
// HBM-bound: 4 B read and 2 B written per element; each thread converts 8
// consecutive elements (two 16-byte loads, one 16-byte store), grid-strided.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kConvertThreads = 256;

__global__ void __launch_bounds__(kConvertThreads)
    convert_kernel(const float* __restrict__ acc, int64_t n8, uint16_t* __restrict__ out) {
  pdl_wait();
  pdl_launch_dependents();
  for (int64_t v = blockIdx.x * static_cast<int64_t>(kConvertThreads) + threadIdx.x; v < n8;
       v += static_cast<int64_t>(gridDim.x) * kConvertThreads) {
    const float4* src = reinterpret_cast<const float4*>(acc + v * 8);
    const float4 a = __ldcs(src), b = __ldcs(src + 1);
    uint4 o;
    o.x = pack_bf16x2(a.x, a.y);
    o.y = pack_bf16x2(a.z, a.w);
    o.z = pack_bf16x2(b.x, b.y);
    o.w = pack_bf16x2(b.z, b.w);
    *reinterpret_cast<uint4*>(out + v * 8) = o;
  }
}

}  // namespace

cudaError_t launch_convert(const float* acc, int64_t n, uint16_t* out, int num_sms, cudaStream_t stream,
                           int* launches) {
  const int64_t n8 = n / 8;  // n = T * d, d a multiple of 64
  int64_t blocks = (n8 + kConvertThreads - 1) / kConvertThreads;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  ++*launches;
  return launch_pdl(convert_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kConvertThreads), 0, stream, acc, n8,
                    out);
}

}  // namespace moe
