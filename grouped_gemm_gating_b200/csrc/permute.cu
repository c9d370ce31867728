// Token rows in expert-sorted order for the paired gate/up GEMM and the
// backward's GEMMs.
//
// x_sorted[p] = x[sorted_token_ids[p] // k] for every live padded row p --
// the row gather of the fused-moe-kernel page's "Grouped GEMM Structure"
// (a[sorted_token_ids // top_k], "Common Pitfalls" 1) and the permuted input
// of the axolotl `_moe_triton_forward` (src/axolotl/monkeypatch/deepseek_v3/
// __init__.py) -- and x_sorted[ntpp + t] = x[t] for the shared expert's
// rows.  Padding rows are left as they are (the forward's GEMM rows they
// feed are never read back) or, for the backward, whose weight gradients
// sum over every row of an expert's blocks, set to zero.  With the rows
// materialised, the GEMMs can load their token operand by TMA like their
// weights.
//
// HBM-bound copy: one warp per row, 16 bytes per lane per step.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kPermuteThreads = 256;

__global__ void __launch_bounds__(kPermuteThreads)
    permute_rows_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ sorted_ids,
                        const int32_t* __restrict__ ntpp_ptr, int T, int k, int S, int d, int P_max,
                        int n_shared_rows, int zero_pad, uint16_t* __restrict__ x_sorted) {
  pdl_wait();
  pdl_launch_dependents();
  int ntpp = *ntpp_ptr;
  if (ntpp < 0) ntpp = 0;
  if (ntpp > P_max) ntpp = P_max;
  const int rows = ntpp + n_shared_rows;
  const int lane = threadIdx.x % kWarp;
  const int nvec = d / 8;  // 16-byte vectors per row
  for (int p = (blockIdx.x * kPermuteThreads + threadIdx.x) / kWarp; p < rows;
       p += gridDim.x * (kPermuteThreads / kWarp)) {
    int tok;
    if (p < ntpp) {
      const int slot = sorted_ids[p];
      tok = static_cast<unsigned>(slot) < static_cast<unsigned>(S) ? slot / k : -1;  // -1: padding
    } else {
      tok = p - ntpp;
      if (tok >= T) tok = -1;
    }
    uint4* dst = reinterpret_cast<uint4*>(x_sorted + static_cast<size_t>(p) * d);
    if (tok < 0) {
      if (zero_pad)
        for (int v = lane; v < nvec; v += kWarp) dst[v] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(tok) * d);
    for (int v = lane; v < nvec; v += kWarp) dst[v] = __ldg(src + v);
  }
}

}  // namespace

cudaError_t launch_permute_rows(const uint16_t* x, const int32_t* sorted_ids, const int32_t* ntpp, int T, int k,
                                int d, int P_max, int n_shared_rows, uint16_t* x_sorted, int num_sms,
                                cudaStream_t stream, int* launches, bool zero_pad) {
  const int64_t rows = static_cast<int64_t>(P_max) + n_shared_rows;
  int64_t blocks = (rows + (kPermuteThreads / kWarp) - 1) / (kPermuteThreads / kWarp);
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  ++*launches;
  return launch_pdl(permute_rows_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kPermuteThreads), 0, stream, x,
                    sorted_ids, ntpp, T, k, T * k, d, P_max, n_shared_rows, zero_pad ? 1 : 0, x_sorted);
}

}  // namespace moe
