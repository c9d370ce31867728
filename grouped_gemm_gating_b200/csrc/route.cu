// Top-k gating over router logits: one warp per token.
//
// Step 1 of "Token-Expert Routing" on the fused-moe-kernel page ("Fused MoE
// Kernel Optimization", skillmd zjli2013): select k experts per token.  The
// grouped variant restricts the choice to the topk_group best of n_group
// contiguous expert groups, as configured by n_group / topk_group in the
// DeepSeek-V3 builder of the axolotl vendor-moe diff
// (scripts/benchmarks/build_deepseek_v3_8b.py, build_config), whose
// norm_topk_prob and routed_scaling_factor give the weight options.
//
// Lane l holds the logits of experts l, l+32, l+64, ... in registers.  The
// selection compares fp32 logits exactly, key (logit descending, expert id
// ascending), so it matches any exact reference bit for bit; the group
// score "top2" is one fp32 addition of the two largest logits of the group.
// Weights: exp(l_j - max) in fp32, summed with a fixed shuffle tree, divided,
// times routed_scaling.
#include "route_impl.cuh"

namespace moe {

namespace {

constexpr int kWarpsPerBlock = 8;

template <int VPL>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    route_kernel(const float* __restrict__ logits, int T, int E, int k, int n_group, int topk_group,
                 int group_score, int renormalize, float routed_scaling, int32_t* __restrict__ topk_ids,
                 float* __restrict__ topk_weights, int32_t* status) {
  __shared__ float s_gscore[kWarpsPerBlock][MOE_MAX_EXPERTS];
  __shared__ unsigned char s_gkeep[kWarpsPerBlock][MOE_MAX_EXPERTS];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int t = blockIdx.x * kWarpsPerBlock + warp;
  pdl_wait();
  pdl_launch_dependents();
  if (t >= T) return;
  route_one_token<VPL>(logits + static_cast<size_t>(t) * E, E, k, n_group, topk_group, group_score, renormalize,
                       routed_scaling, s_gscore[warp], s_gkeep[warp], topk_ids + static_cast<size_t>(t) * k,
                       topk_weights + static_cast<size_t>(t) * k, status, lane);
}

}  // namespace

cudaError_t launch_route(const float* logits, int T, int E, int k, int n_group, int topk_group, int group_score,
                         int renormalize, float routed_scaling, int32_t* topk_ids, float* topk_weights,
                         int32_t* status, cudaStream_t stream, int* launches) {
  const int grid = (T + kWarpsPerBlock - 1) / kWarpsPerBlock;
  const int block = kWarpsPerBlock * 32;
  auto kern = E <= 32 ? route_kernel<1> : E <= 64 ? route_kernel<2> : E <= 128 ? route_kernel<4> : route_kernel<8>;
  cudaError_t err = launch_pdl(kern, dim3(grid), dim3(block), 0, stream, logits, T, E, k, n_group, topk_group,
                               group_score, renormalize, routed_scaling, topk_ids, topk_weights, status);
  ++*launches;
  return err;
}

}  // namespace moe
