// Per-token top-k gating, shared by the routing kernel and the fused
// route+align kernel.  See route.cu for the method and its sources.
#pragma once
#include <cmath>

#include "common.cuh"

namespace moe {
namespace route_detail {

// Unsigned key with the order of the fp32 values (-0 taken as +0, so the
// two zeros tie as they do in a float comparison); 0 is below every value
// and marks an excluded expert.
__device__ __forceinline__ uint32_t order_key(float v) {
  uint32_t u = __float_as_uint(v);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
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

  // k rounds of warp arg-max over the remaining allowed experts, on
  // order-preserving integer keys: one warp max of the lanes' best keys,
  // then one warp min of the expert ids that hold it (ties -> lowest id).
  uint32_t key[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) key[i] = allowed[i] ? order_key(v[i]) : 0u;
  int my_id = 0;
  float my_val = 0.0f;
  for (int j = 0; j < k; ++j) {
    uint32_t hk = 0u;
    int hi = 0;
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if (key[i] > hk) {  // strict: the lowest id of this lane among equal keys
        hk = key[i];
        hi = i;
      }
    const uint32_t m = __reduce_max_sync(0xffffffffu, hk);
    const uint32_t cand = (hk == m && hk != 0u) ? static_cast<uint32_t>(lane + 32 * hi) : 0xffffffffu;
    const uint32_t win = __reduce_min_sync(0xffffffffu, cand);
    if (static_cast<int>(win & 31u) == lane) {
#pragma unroll
      for (int i = 0; i < VPL; ++i)
        if (i == static_cast<int>(win >> 5)) key[i] = 0u;
    }
    if (lane == j) {
      my_id = static_cast<int>(win);
      my_val = key_value(m);
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
