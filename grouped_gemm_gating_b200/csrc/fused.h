// Host-visible interface of the fused expert kernel (gate/up GEMM + act,
// down GEMM + top-k weight, optional scatter-reduce) for block_m <= 64.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace moe {

struct FusedArgs {
  CUtensorMap tm_w13;   // routed gate/up (or fc1) weights, 3-D {d, N1, E}, 128-row boxes
  CUtensorMap tm_w13s;  // shared expert, 3-D {d, N1, 1}
  CUtensorMap tm_w2;    // routed down weights, 3-D {F, d, E}, 128-row boxes
  CUtensorMap tm_w2s;   // shared expert, 3-D {F, d, 1}
  const uint16_t* x;    // [T, d] bf16
  uint16_t* h;          // [P_total, F] bf16 (workspace)
  float* y;             // [P_total, d] fp32 (workspace)
  uint16_t* out;        // [T, d] bf16
  const int32_t* sorted_ids;
  const int32_t* expert_ids;
  const int32_t* ntpp;
  const int32_t* inv_pos;
  const float* topk_w;  // [T * k]
  // Cross-CTA counters, zero on entry; the last CTA to finish resets them.
  int32_t* ready;       // [blocks]   gate/up tiles published per block
  int32_t* done;        // [d tiles]  down tiles finished per d-column tile
  int32_t* finished;    // [1]        CTAs that have finished
  int32_t* status;
  int T, k, S, E, d, F;
  int block_m;
  int max_routed_blocks;
  int n_shared_blocks;
  int do_combine;       // 1: the kernel also writes out (fused_expert_combines)
};

bool fused_expert_supported(int block_m);
// True when the fused kernel also does the scatter-reduce (T*k <= 64, no shared expert).
bool fused_expert_combines(int T, int k, int n_shared);
cudaError_t launch_fused_expert(int act_epi, int block_m, const FusedArgs& args, int grid, cudaStream_t stream);

}  // namespace moe
