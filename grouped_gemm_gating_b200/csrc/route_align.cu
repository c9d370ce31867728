// Route and align in one launch for small batches (decode / verifier shapes).
//
// The two first steps of the fused-moe-kernel page's "Token-Expert Routing"
// (top-k gating, then sort by expert and pad to BLOCK_SIZE_M), done by one
// 1024-thread block: each warp routes tokens with the same per-token code as
// the routing kernel, the chosen ids stay in shared memory, and the block
// then runs the same stable counting sort as the single-block align kernel.
// For a handful of tokens both steps are pure latency, so one launch instead
// of two is the saving; results are bit-identical to the two-kernel path.
#include "align_impl.cuh"
#include "route_impl.cuh"

namespace moe {

namespace {

constexpr int kFusedMaxT = 64;
constexpr int kFusedMaxS = 1024;
constexpr int kFusedMaxGroups = 64;

// NWARPS warps: 8 for up to 256 slots (decode), 32 above.
template <int VPL, int NWARPS>
__global__ void __launch_bounds__(NWARPS * 32)
    route_align_kernel(const float* __restrict__ logits, int T, int E, int k, int n_group, int topk_group,
                       int group_score, int renormalize, float routed_scaling, int32_t* __restrict__ topk_ids,
                       float* __restrict__ topk_weights, int bm, int P_max, int32_t* __restrict__ sorted_ids,
                       int32_t* __restrict__ expert_ids, int32_t* ntpp, int32_t* __restrict__ inv_pos,
                       int32_t* status) {
  __shared__ int s_ids[kFusedMaxS];
  __shared__ int cnt[MOE_MAX_EXPERTS];
  __shared__ int off[MOE_MAX_EXPERTS + 1];
  __shared__ int run[MOE_MAX_EXPERTS];
  __shared__ int tot[MOE_MAX_EXPERTS];
  constexpr int kFusedWarps = NWARPS;
  constexpr int kFusedThreads = NWARPS * 32;
  __shared__ int wcnt[kFusedWarps][MOE_MAX_EXPERTS];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // While routing, each warp's row of wcnt doubles as its group-score
  // scratch (64 floats, then 64 keep flags); it is zeroed before the align.
  float* gscore = reinterpret_cast<float*>(&wcnt[warp][0]);
  unsigned char* gkeep = reinterpret_cast<unsigned char*>(&wcnt[warp][kFusedMaxGroups]);
  pdl_wait();
  pdl_launch_dependents();
  for (int t = warp; t < T; t += kFusedWarps) {
    const int id = route_one_token<VPL>(logits + static_cast<size_t>(t) * E, E, k, n_group, topk_group, group_score,
                                        renormalize, routed_scaling, gscore, gkeep,
                                        topk_ids + static_cast<size_t>(t) * k, topk_weights + static_cast<size_t>(t) * k,
                                        status, lane);
    if (lane < k) s_ids[t * k + lane] = id;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kFusedWarps * MOE_MAX_EXPERTS; i += kFusedThreads) (&wcnt[0][0])[i] = 0;
  const int S = T * k;
  auto get_expert = [&](int s, bool) { return s_ids[s]; };
  align_detail::align_one_block<kFusedWarps>(get_expert, S, E, bm, P_max, sorted_ids, expert_ids, ntpp, inv_pos, cnt,
                                             off, run, tot, wcnt);
}

}  // namespace

bool route_align_fusable(int T, int k, int n_group) {
  return T <= kFusedMaxT && T * k <= kFusedMaxS && n_group <= kFusedMaxGroups;
}

cudaError_t launch_route_align(const float* logits, int T, int E, int k, int n_group, int topk_group,
                               int group_score, int renormalize, float routed_scaling, int32_t* topk_ids,
                               float* topk_weights, int block_m, int P_max, int32_t* sorted_ids, int32_t* expert_ids,
                               int32_t* ntpp, int32_t* inv_pos, int32_t* status, cudaStream_t stream,
                               int* launches) {
  const bool small = T * k <= 256;
  auto kern = small ? (E <= 32    ? route_align_kernel<1, 8>
                       : E <= 64  ? route_align_kernel<2, 8>
                       : E <= 128 ? route_align_kernel<4, 8>
                                  : route_align_kernel<8, 8>)
                    : (E <= 32    ? route_align_kernel<1, 32>
                       : E <= 64  ? route_align_kernel<2, 32>
                       : E <= 128 ? route_align_kernel<4, 32>
                                  : route_align_kernel<8, 32>);
  ++*launches;
  return launch_pdl(kern, dim3(1), dim3(small ? 256 : 1024), 0, stream, logits, T, E, k, n_group, topk_group, group_score,
                    renormalize, routed_scaling, topk_ids, topk_weights, block_m, P_max, sorted_ids, expert_ids, ntpp,
                    inv_pos, status);
}

}  // namespace moe
