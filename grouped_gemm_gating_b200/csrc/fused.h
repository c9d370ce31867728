// Host-visible interface of the fused expert kernel for block_m <= 64: the
// gate/up GEMM with its activation, the down GEMM split along d_ff with the
// top-k weights, and the scatter-reduce, in one persistent launch.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace moe {

// Routing done inside the fused kernel (small batches): every CTA routes all
// tokens and sorts their slots in shared memory; CTA 0 also writes the
// results to these outputs, which then equal moe_route + moe_align's.
struct FusedRoute {
  const float* logits;  // [T, E] fp32
  int n_group, topk_group, group_score, renormalize;
  float routed_scaling;
  int32_t* topk_ids;    // [T, k] out
  float* topk_w;        // [T, k] out
  int32_t* sorted_ids;  // [P_max] out
  int32_t* expert_ids;  // [P_max / block_m] out
  int32_t* ntpp;        // [1] out
  int32_t* inv_pos;     // [T * k] out
  int P_max;
};

struct FusedArgs {
  CUtensorMap tm_w13;   // routed gate/up (or fc1) weights, 3-D {d, N1, E}; boxes of 64 x 64 rows
                        // (SwiGLU: 64 gate rows, then the matching 64 up rows) or 64 x 128 (relu^2)
                        // fp8 weights: uint8 e4m3, boxes of 64 x 128 rows, no swizzle
  CUtensorMap tm_w13s;  // shared expert, 3-D {d, N1, 1}, same boxes
  CUtensorMap tm_w2;    // routed down weights, 3-D {F, d, E}, 64 x 128 boxes (fp8: the same, uint8)
  CUtensorMap tm_w2s;   // shared expert, 3-D {F, d, 1}
  // fp8 weights only: the power-of-two scale bytes, K-block-major
  // [E, K / 32, rows] as 3-D {rows, K / 32, E} maps with 128 x 2 boxes (the
  // scales of one stage's 128 rows and 64 K values)
  CUtensorMap tm_s13, tm_s13s, tm_s2, tm_s2s;
  const uint16_t* x;    // [T, d] bf16
  float* acc;           // [T, d] fp32 accumulator (workspace; zeroed by the kernel)
  uint16_t* out;        // [T, d] bf16
  const int32_t* sorted_ids;
  const int32_t* expert_ids;
  const int32_t* ntpp;
  const float* topk_w;  // [T * k]
  int32_t* sync;        // [3] grid counters: CTAs that zeroed their accumulator slice, CTAs
                        // finished (both zero at rest), release generation (any value)
  int32_t* status;
  uint64_t wait_ns;     // limit of every pipeline and grid wait (kWaitLimitNs unless lowered for a test)
  int start_surplus;    // extra arrivals the start barrier waits for (0; > 0 only in the timeout test)
  int T, k, S, E, d, F;
  int block_m;
  int max_routed_blocks;
  int n_shared_blocks;
  FusedRoute route;     // used by the launch with in-kernel routing only
};

// Rows per TMA box of the fused kernel's weight tensor maps.  A stage of 128
// weight rows (gate, up or fc1 rows of one 64-wide K block, or W2 rows) is
// filled by several boxes.  Boxes shorter than a stage streamed faster on the
// decode shape; 16-row boxes were far slower.
constexpr int kFusedBoxRowsGated = 32;
constexpr int kFusedBoxRowsRelu2 = 64;
constexpr int kFusedBoxRowsW2 = 64;

bool fused_expert_supported(int block_m);
// In-kernel routing covers block_m = 16, T*k <= 256, n_group <= 64.
bool fused_routing_supported(int T, int k, int E, int n_group, int block_m);
// Upper bound on the fused kernel's tiles, for grid sizing.
int64_t fused_expert_max_tiles(int act_epi, int total_blocks_max, int F);
cudaError_t launch_fused_expert(int act_epi, int block_m, bool route, const FusedArgs& args, int grid,
                                cudaStream_t stream, bool fp8 = false);

}  // namespace moe
