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
#include <cmath>

#include "common.cuh"

namespace moe {

namespace {

struct Cand {
  float v;
  int i;
};

// true if a is selected before b
__device__ __forceinline__ bool beats(const Cand& a, const Cand& b) {
  return a.v > b.v || (a.v == b.v && a.i < b.i);
}

__device__ __forceinline__ Cand warp_best(Cand c) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    Cand o;
    o.v = __shfl_xor_sync(0xffffffffu, c.v, off);
    o.i = __shfl_xor_sync(0xffffffffu, c.i, off);
    if (beats(o, c)) c = o;
  }
  return c;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

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

  const float* row = logits + static_cast<size_t>(t) * E;
  float v[VPL];
  bool allowed[VPL];
  bool finite = true;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? row[e] : -INFINITY;
    allowed[i] = e < E;
    if (e < E && !isfinite(v[i])) finite = false;
  }
  if (__any_sync(0xffffffffu, !finite) && lane == 0) set_status(status, MOE_ERR_NONFINITE);

  if (n_group > 1) {
    const int gsize = E / n_group;
    for (int g = 0; g < n_group; ++g) {
      // top-2 of the group over this lane's experts, then across the warp
      float a = -INFINITY, b = -INFINITY;
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E && e / gsize == g) {
          if (v[i] > a) {
            b = a;
            a = v[i];
          } else if (v[i] > b) {
            b = v[i];
          }
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float oa = __shfl_xor_sync(0xffffffffu, a, off);
        const float ob = __shfl_xor_sync(0xffffffffu, b, off);
        // merge two sorted pairs into the top-2 of the four values
        const float hi = fmaxf(a, oa);
        const float lo = fmaxf(fminf(a, oa), fmaxf(b, ob));
        a = hi;
        b = lo;
      }
      float score = a;
      if (group_score == MOE_GROUP_TOP2SUM && gsize >= 2) score = __fadd_rn(a, b);
      if (lane == 0) s_gscore[warp][g] = score;
    }
    __syncwarp();
    // group g is kept if fewer than topk_group groups beat it
    for (int g = lane; g < n_group; g += 32) {
      const float sg = s_gscore[warp][g];
      int better = 0;
      for (int h = 0; h < n_group; ++h) {
        const float sh = s_gscore[warp][h];
        better += (sh > sg || (sh == sg && h < g)) ? 1 : 0;
      }
      s_gkeep[warp][g] = better < topk_group ? 1 : 0;
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E) allowed[i] = s_gkeep[warp][e / gsize] != 0;
    }
  }

  // k rounds of warp arg-max over the remaining allowed experts
  int my_id = 0;
  float my_val = 0.0f;
  for (int j = 0; j < k; ++j) {
    Cand best{-INFINITY, 0x7fffffff};
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const Cand c{v[i], lane + 32 * i};
      if (allowed[i] && (best.i == 0x7fffffff || beats(c, best))) best = c;
    }
    best = warp_best(best);
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if (lane + 32 * i == best.i) allowed[i] = false;
    if (lane == j) {
      my_id = best.i;
      my_val = best.v;
    }
  }

  float w;
  if (renormalize) {
    const float m = __shfl_sync(0xffffffffu, my_val, 0);  // first pick is the largest chosen logit
    const float ex = lane < k ? expf(my_val - m) : 0.0f;
    const float z = warp_sum(ex);
    w = ex / z;
  } else {
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < VPL; ++i) m = fmaxf(m, v[i]);
    m = warp_max(m);
    float part = 0.0f;
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if (lane + 32 * i < E) part += expf(v[i] - m);
    const float z = warp_sum(part);
    w = expf(my_val - m) / z;
  }
  if (lane < k) {
    topk_ids[static_cast<size_t>(t) * k + lane] = my_id;
    topk_weights[static_cast<size_t>(t) * k + lane] = w * routed_scaling;
  }
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
