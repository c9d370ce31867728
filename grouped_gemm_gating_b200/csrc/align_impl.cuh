// Building blocks of the stable counting sort of token-slots by expert,
// shared by the align kernels and the fused route+align kernel.  See
// align.cu for the method and its sources.
#pragma once
#include "common.cuh"

namespace moe {
namespace align_detail {

__device__ __forceinline__ int load_expert(const int32_t* ids, int s, int S, int E, int32_t* status) {
  if (s >= S) return -1;
  const int e = ids[s];
  if (e < 0 || e >= E) {
    set_status(status, MOE_ERR_BAD_EXPERT_ID);
    return -1;
  }
  return e;
}

// Exclusive prefix of padded counts over experts, by one warp.  off[E] is
// the padded total.  bm is a power of two (block_m, or 1 for no padding), so
// rounding up is a mask: a runtime integer division per expert made this
// scan cost more than a microsecond.
__device__ __forceinline__ void warp_padded_scan(const int* cnt, int* off, int E, int bm, int lane) {
  constexpr int kPer = MOE_MAX_EXPERTS / 32;
  int local[kPer];
  int sum = 0;
  const int mask = -bm;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = lane * kPer + i;
    const int c = e < E ? cnt[e] : 0;
    local[i] = (c + bm - 1) & mask;
    sum += local[i];
  }
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  int run = incl - sum;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = lane * kPer + i;
    if (e < E) off[e] = run;
    run += local[i];
  }
  if (lane == 31) off[E] = incl;
}

// Block b (rows [b*bm, (b+1)*bm)) belongs to the expert e with
// off[e] <= b*bm < off[e+1]; -1 past the padded total.
__device__ __forceinline__ int block_expert(const int* off, int E, int p) {
  if (p >= off[E]) return -1;
  int lo = 0, hi = E - 1;  // last e with off[e] <= p
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= p)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

// One round of the stable scatter over `nthreads` consecutive slots.  wcnt
// is [nwarps][E] of zeros on entry and on exit; run[e] is advanced.
template <int NWARPS>
__device__ __forceinline__ void scatter_round(int e, int s, int (*wcnt)[MOE_MAX_EXPERTS], int* run, int* tot, int E,
                                              int32_t* sorted_ids, int32_t* inv_pos) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int rank = __popc(peers & ((1u << lane) - 1u));
  if (e >= 0 && rank == 0) wcnt[warp][e] = __popc(peers);
  __syncthreads();
  if (threadIdx.x < E) {
    int acc = 0;
#pragma unroll 4
    for (int w = 0; w < NWARPS; ++w) {
      const int c = wcnt[w][threadIdx.x];
      wcnt[w][threadIdx.x] = acc;
      acc += c;
    }
    tot[threadIdx.x] = acc;
  }
  __syncthreads();
  if (e >= 0) {
    const int pos = run[e] + wcnt[warp][e] + rank;
    sorted_ids[pos] = s;
    inv_pos[s] = pos;
  }
  __syncthreads();
  if (threadIdx.x < E) {
    run[threadIdx.x] += tot[threadIdx.x];
#pragma unroll 4
    for (int w = 0; w < NWARPS; ++w) wcnt[w][threadIdx.x] = 0;
  }
  __syncthreads();
}

// The whole align in one thread block of NWARPS warps: histogram, padded
// scan, padding fill, block experts, stable scatter.  get_expert(s) returns
// slot s's expert (or -1 to skip it); shared scratch is passed in: cnt, run,
// tot [E], off [E+1], wcnt [NWARPS][MOE_MAX_EXPERTS] (zero on entry).
template <int NWARPS, typename GetExpert>
__device__ __forceinline__ void align_one_block(GetExpert get_expert, int S, int E, int bm, int P_max,
                                                int32_t* __restrict__ sorted_ids, int32_t* __restrict__ expert_ids,
                                                int32_t* ntpp, int32_t* __restrict__ inv_pos, int* cnt, int* off,
                                                int* run, int* tot, int (*wcnt)[MOE_MAX_EXPERTS]) {
  constexpr int kThreads = NWARPS * 32;
  const int tid = threadIdx.x;
  for (int i = tid; i < E; i += kThreads) cnt[i] = 0;
  __syncthreads();
  for (int s = tid; s < S; s += kThreads) {
    const int e = get_expert(s, true);
    if (e >= 0) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  if (tid < 32) warp_padded_scan(cnt, off, E, bm, tid);
  __syncthreads();
  if (tid < E) run[tid] = off[tid];
  if (tid == 0) *ntpp = off[E];
  for (int p = tid; p < P_max; p += kThreads) sorted_ids[p] = S;
  for (int b = tid; b < P_max / bm; b += kThreads) expert_ids[b] = block_expert(off, E, b * bm);
  __syncthreads();
  for (int base = 0; base < S; base += kThreads) {
    const int s = base + tid;
    const int e = s < S ? get_expert(s, false) : -1;
    scatter_round<NWARPS>(e, s, wcnt, run, tot, E, sorted_ids, inv_pos);
  }
}

}  // namespace align_detail
}  // namespace moe
