// Host-visible interface of the tcgen05 grouped GEMM kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace moe {

enum EpiKind : int {
  kEpiSwiGLU = 0,      // gate/up GEMM, h = silu(gate) * up
  kEpiRelu2 = 1,       // fc1 GEMM, h = max(a, 0)^2
  kEpiScale = 2,       // down GEMM, acc[token] += topk_weight(row) * row result (fp32)
  kEpiRouter = 3,      // router GEMM, logits = x . W_g^T (fp32)
  // backward (token rows by TMA from the expert-sorted copies)
  kEpiPreSwiGLU = 4,   // gate/up pre-activations [g | u] of every row, fp32
  kEpiPreRelu2 = 5,    // fc1 pre-activations, fp32
  kEpiGradSwiGLU = 6,  // dh = W2^T dout rows (W2 read MN-major); epilogue: [dg | du] from [g | u] (bf16),
                       // w * h, and dL/dw of the row's slot
  kEpiGradRelu2 = 7,   // the same for relu^2: da over a
  kEpiDx = 8           // dx rows = da . W13 (W13 read MN-major), added into the fp32 accumulator
};

// Arguments of one grouped GEMM launch (token-major tiles, block_m = 128).
// Rows of the token operand are the
// padded positions p = blk * block_m + r of the expert-sorted layout; block
// blk < routed_blocks belongs to expert expert_ids[blk], blocks after that
// (n_shared_blocks of them) to the shared expert, whose token is
// (blk - routed_blocks) * block_m + r.
struct GemmArgs {
  CUtensorMap tm_w;   // routed expert weights, 3-D {K, rows per expert, E}, 128B swizzle
  CUtensorMap tm_ws;  // shared expert weights, 3-D {K, rows, 1}
  CUtensorMap tm_x;   // down GEMM only: h, 2-D {K, P_total} with 64 x block_m boxes
  const uint16_t* x;  // gate/up GEMM only: token rows gathered from x [T, K]
  const int32_t* sorted_ids;
  const int32_t* expert_ids;
  const int32_t* ntpp;
  const float* topk_w;  // [T * k], indexed by slot
  void* out;            // gate/up GEMM: bf16 h [P_total, n_out]
  float* acc;           // fp32 [T, d] accumulator: zeroed by the gate/up GEMM, reduced into by the down GEMM
  int64_t acc_elems;    // T * d
  int32_t* status;
  uint64_t wait_ns;     // limit of every pipeline wait (kWaitLimitNs unless lowered for a test)
  int tfull_surplus;    // extra arrivals the accumulator-full barriers expect (0; > 0 only in the timeout test)
  int T, k, S, E;
  int K;                // reduction length (multiple of 64)
  int n_out;            // output columns (multiple of 16)
  int up_row_offset;    // SwiGLU: first up-projection row of an expert (= F)
  int block_m;
  int max_routed_blocks;
  int n_shared_blocks;
  int pass_cols;        // output-column tiles per pass of the tile walk (0: one pass)
  // backward only
  int out_ld;           // row stride (elements) of `out` and `pre` (pre / grad kinds: n1)
  const float* pre;     // grad kinds: the fp32 pre-activations [P_total, n1] (`out` is then da, bf16)
  uint16_t* hw;         // grad kinds: w * h [P_total, F] bf16
  float* dtopk;         // grad kinds: dL/d topk_weights [T * k] (fp32 adds; zeroed by the pre kinds)
  float* zero2;         // pre kinds: a second buffer their spare warp zeroes (dtopk), zero2_elems floats
  int64_t zero2_elems;
  // router GEMM only: fp32 logits [T, E]
  float* logits;
};

// Rows of one weight TMA box (= output columns of one tile) for an epilogue.
int gemm_box_rows(int epi);
// Upper bound on tiles of one launch, for grid sizing.
int64_t gemm_max_tiles(int epi, int max_routed_blocks, int n_shared_blocks, int n_out);
cudaError_t launch_grouped_gemm(int epi, const GemmArgs& args, int grid, cudaStream_t stream);
// Router GEMM: x [T, K] (tm_x, 2-D {K, T}, 64 x 128 boxes) times W_g [E, K]
// (tm_ws, 3-D {K, E, 1}, 256-row boxes), E <= 256; the routing kernel gates
// the logits it writes (top-k k <= 16).
constexpr int kRouterMaxE = 256;
constexpr int kRouterMaxK = 16;

// The same GEMMs on CTA pairs (cluster of two, tcgen05 cta_group::2): args
// as for launch_grouped_gemm, except that tm_w / tm_ws use 128-row boxes and
// the gate/up GEMM reads its token rows through tm_x (permuted x, 2-D
// {K, P_total}, 64 x 128 boxes) instead of gathering them.
bool gemm_pair_supported(int block_m, int total_blocks_max);
cudaError_t launch_grouped_gemm_pair(int epi, const GemmArgs& args, int grid, cudaStream_t stream);

// The gate/up (fc1) GEMM with gathered token rows on units of two 128-row
// blocks of one expert (256-token tiles sharing each weight stage): args as
// for launch_grouped_gemm; at most kWideMaxBlocks blocks per launch.
constexpr int kWideMaxBlocks = 8192;
bool gemm_wide_supported(int epi, int block_m, int total_blocks_max);
cudaError_t launch_grouped_gemm_wide(int epi, const GemmArgs& args, int grid, cudaStream_t stream);

// Per-expert weight gradient (backward): for every expert e (and the shared
// expert, when present), dW_e [M, N] = sum over the rows p of e's blocks of
// A[p, :]^T B[p, :], with A [P_total, M] and B [P_total, N] in the
// expert-sorted row order (padding rows zero), rounded to bf16.  Both
// operands are read MN-major (their M / N index contiguous) by TMA.
struct WgradArgs {
  CUtensorMap tm_a;        // A, 2-D {M, P_total}, 64 x 64 boxes, 128B swizzle
  CUtensorMap tm_b;        // B, 2-D {N, P_total}, 64 x 64 boxes, 128B swizzle
  const int32_t* expert_ids;
  const int32_t* ntpp;
  uint16_t* out;           // [E, M, N] bf16
  uint16_t* out_shared;    // [M, N] bf16 (the shared expert's rows follow the routed ones)
  int32_t* status;
  uint64_t wait_ns;
  int E, M, N;
  int block_m;             // 128
  int max_routed_blocks;
  int n_shared_blocks;
};
int64_t wgrad_max_tiles(int E, int n_shared, int M, int N);
cudaError_t launch_wgrad(const WgradArgs& args, int grid, cudaStream_t stream);

}  // namespace moe
