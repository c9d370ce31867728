// Sort token-slots by expert and pad every expert to a multiple of block_m.
//
// Steps 2-3 of "Token-Expert Routing" and the indirection arrays of
// "Grouped GEMM Structure" on the fused-moe-kernel page ("Fused MoE Kernel
// Optimization", skillmd zjli2013): sorted_token_ids (slot ids s = t*k + j,
// so that s // top_k is the token, "Common Pitfalls" 1), expert_ids (one
// expert per block), num_tokens_post_padded, and padding ids equal to
// S = T*k, i.e. at least num_valid_tokens ("Common Pitfalls" 2).  The
// per-expert counts rounded up to the alignment and their running offsets
// play the role of m_sizes / write_offsets in the axolotl vendor-moe diff
// (src/axolotl/kernels/moe/indices/indices.py, generate_permute_indices),
// except that an expert with no slot gets no block.
//
// The sort is a stable counting sort: within an expert, slots keep their
// ascending order, so the result is unique and both code paths below give
// the same bits.
//   * S <= kSingleBlockMax: one 1024-thread block does histogram, scan,
//     padding fill and the stable scatter in one launch (decode latency).
//   * larger S: per-chunk histograms (one block per chunk), then per chunk
//     one block that scans all chunks' counts itself and places its slots
//     (stable scatter).
// Within a round of slots, the rank of a slot among equal experts comes from
// __match_any_sync inside the warp plus an exclusive prefix over the warps.
#include "align_impl.cuh"

namespace moe {

namespace {

using namespace align_detail;

constexpr int kSingleBlockMax = 8192;
constexpr int kSmallThreads = 1024;
constexpr int kChunk = 2048;        // slots per chunk on the multi-block path
constexpr int kChunkThreads = 256;  // threads per chunk block (count)
constexpr int kScatterThreads = 1024;  // threads per chunk block (scatter: two rounds of 1024 slots)

__global__ void __launch_bounds__(kSmallThreads)
    align_single_kernel(const int32_t* __restrict__ ids, int S, int E, int bm, int P_max,
                        int32_t* __restrict__ sorted_ids, int32_t* __restrict__ expert_ids, int32_t* ntpp,
                        int32_t* __restrict__ inv_pos, int32_t* status) {
  constexpr int kWarps = kSmallThreads / 32;
  __shared__ int cnt[MOE_MAX_EXPERTS];
  __shared__ int off[MOE_MAX_EXPERTS + 1];
  __shared__ int run[MOE_MAX_EXPERTS];
  __shared__ int tot[MOE_MAX_EXPERTS];
  __shared__ int wcnt[kWarps][MOE_MAX_EXPERTS];
  for (int i = threadIdx.x; i < kWarps * MOE_MAX_EXPERTS; i += kSmallThreads) (&wcnt[0][0])[i] = 0;
  pdl_wait();
  pdl_launch_dependents();
  auto get_expert = [&](int s, bool report) { return load_expert(ids, s, S, E, report ? status : nullptr); };
  align_one_block<kWarps>(get_expert, S, E, bm, P_max, sorted_ids, expert_ids, ntpp, inv_pos, cnt, off, run, tot,
                          wcnt);
}

// ---- multi-block path ----------------------------------------------------

__global__ void __launch_bounds__(kChunkThreads)
    align_count_kernel(const int32_t* __restrict__ ids, int S, int E, int32_t* __restrict__ counts,
                       int32_t* status) {
  __shared__ int cnt[MOE_MAX_EXPERTS];
  const int c = blockIdx.x;
  for (int i = threadIdx.x; i < E; i += kChunkThreads) cnt[i] = 0;
  pdl_wait();
  pdl_launch_dependents();
  __syncthreads();
  const int end = min(S, (c + 1) * kChunk);
  for (int s = c * kChunk + threadIdx.x; s < end; s += kChunkThreads) {
    const int e = load_expert(ids, s, S, E, status);
    if (e >= 0) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < E; i += kChunkThreads) counts[static_cast<size_t>(c) * E + i] = cnt[i];
}

// Every chunk block sums the counts of all chunks itself (per expert: the
// total, and the part in chunks before its own), scans the padded totals
// and so knows where its slots go; it also writes its share of the layout
// (padding ids, block experts) and then places its slots.
__global__ void __launch_bounds__(kScatterThreads)
    align_place_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ counts, int nchunks, int S,
                       int E, int bm, int P_max, int32_t* __restrict__ sorted_ids, int32_t* __restrict__ expert_ids,
                       int32_t* ntpp, int32_t* __restrict__ inv_pos) {
  constexpr int kWarps = kScatterThreads / 32;
  constexpr int kSlices = kScatterThreads / MOE_MAX_EXPERTS;  // contiguous chunk ranges per expert
  __shared__ int part[kSlices][MOE_MAX_EXPERTS];
  __shared__ int before[kSlices][MOE_MAX_EXPERTS];
  __shared__ int cnt[MOE_MAX_EXPERTS];
  __shared__ int off[MOE_MAX_EXPERTS + 1];
  __shared__ int run[MOE_MAX_EXPERTS];
  __shared__ int tot[MOE_MAX_EXPERTS];
  __shared__ int wcnt[kWarps][MOE_MAX_EXPERTS];
  const int c = blockIdx.x;
  const int tid = threadIdx.x;
  const int e = tid % MOE_MAX_EXPERTS, slice = tid / MOE_MAX_EXPERTS;
  const int per = (nchunks + kSlices - 1) / kSlices;
  const int c_lo = slice * per, c_hi = min(nchunks, c_lo + per);
  for (int i = tid; i < kWarps * MOE_MAX_EXPERTS; i += kScatterThreads) (&wcnt[0][0])[i] = 0;
  pdl_wait();
  pdl_launch_dependents();
  // threads over experts (coalesced loads), each summing one chunk range
  int sum = 0, pre = 0;
  if (e < E) {
#pragma unroll 8
    for (int cc = c_lo; cc < c_hi; ++cc) {
      const int v = counts[static_cast<size_t>(cc) * E + e];
      sum += v;
      pre += cc < c ? v : 0;
    }
  }
  part[slice][e] = sum;
  before[slice][e] = pre;
  __syncthreads();
  if (tid < E) {
    int total = 0, b = 0;
#pragma unroll
    for (int s2 = 0; s2 < kSlices; ++s2) {
      total += part[s2][tid];
      b += before[s2][tid];
    }
    cnt[tid] = total;
    tot[tid] = b;
  }
  __syncthreads();
  if (tid < 32) warp_padded_scan(cnt, off, E, bm, tid);
  __syncthreads();
  if (tid < E) run[tid] = off[tid] + tot[tid];
  // this block's share of the layout: padding inside experts' last blocks,
  // the tail past the padded total, the block experts
  if (c == 0 && tid == 0) *ntpp = off[E];
  for (int e2 = c; e2 < E; e2 += gridDim.x)
    for (int p = off[e2] + cnt[e2] + tid; p < off[e2 + 1]; p += kScatterThreads) sorted_ids[p] = S;
  for (int p = off[E] + c * kScatterThreads + tid; p < P_max; p += gridDim.x * kScatterThreads) sorted_ids[p] = S;
  for (int b = c * kScatterThreads + tid; b < P_max / bm; b += gridDim.x * kScatterThreads)
    expert_ids[b] = block_expert(off, E, b * bm);
  __syncthreads();
  const int end = min(S, (c + 1) * kChunk);
  for (int base = c * kChunk; base < end; base += kScatterThreads) {
    const int s = base + tid;
    const int ex = s < end ? load_expert(ids, s, S, E, nullptr) : -1;
    scatter_round<kWarps>(ex, s, wcnt, run, tot, E, sorted_ids, inv_pos);
  }
}

}  // namespace

bool align_uses_single_block(int S) { return S <= kSingleBlockMax; }

int align_num_chunks(int S) { return (S + kChunk - 1) / kChunk; }

cudaError_t launch_align(const int32_t* topk_ids, int S, int E, int block_m, int P_max, int32_t* sorted_ids,
                         int32_t* expert_ids, int32_t* ntpp, int32_t* inv_pos, int32_t* ws, int32_t* status,
                         cudaStream_t stream, int* launches) {
  if (align_uses_single_block(S)) {
    ++*launches;
    return launch_pdl(align_single_kernel, dim3(1), dim3(kSmallThreads), 0, stream, topk_ids, S, E, block_m, P_max,
                      sorted_ids, expert_ids, ntpp, inv_pos, status);
  }
  const int nchunks = align_num_chunks(S);
  int32_t* counts = ws;
  cudaError_t err = launch_pdl(align_count_kernel, dim3(nchunks), dim3(kChunkThreads), 0, stream, topk_ids, S, E,
                               counts, status);
  if (err != cudaSuccess) return err;
  err = launch_pdl(align_place_kernel, dim3(nchunks), dim3(kScatterThreads), 0, stream, topk_ids,
                   static_cast<const int32_t*>(counts), nchunks, S, E, block_m, P_max, sorted_ids, expert_ids, ntpp,
                   inv_pos);
  *launches += 2;
  return err;
}

}  // namespace moe
