// Per-token top-k gating, shared by the routing kernel and the fused
// route+align kernel.  See route.cu for the method and its sources.
#pragma once
#include <cmath>

#include "common.cuh"

namespace moe {
namespace route_detail {

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

}  // namespace route_detail

// Routes one token with one full warp.  Lane l holds experts l, l+32, ...
// gscore / gkeep: per-warp scratch of at least n_group entries (used only
// when n_group > 1).  Lane j < k writes ids_out[j], w_out[j] and returns its
// expert id (other lanes return an unspecified value).
template <int VPL>
__device__ __forceinline__ int route_one_token(const float* __restrict__ row, int E, int k, int n_group,
                                               int topk_group, int group_score, int renormalize,
                                               float routed_scaling, float* gscore, unsigned char* gkeep,
                                               int32_t* ids_out, float* w_out, int32_t* status, int lane) {
  using namespace route_detail;
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
      if (lane == 0) gscore[g] = score;
    }
    __syncwarp();
    // group g is kept if fewer than topk_group groups beat it
    for (int g = lane; g < n_group; g += 32) {
      const float sg = gscore[g];
      int better = 0;
      for (int h = 0; h < n_group; ++h) {
        const float sh = gscore[h];
        better += (sh > sg || (sh == sg && h < g)) ? 1 : 0;
      }
      gkeep[g] = better < topk_group ? 1 : 0;
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E) allowed[i] = gkeep[e / gsize] != 0;
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
    ids_out[lane] = my_id;
    w_out[lane] = w * routed_scaling;
  }
  return my_id;
}

}  // namespace moe
