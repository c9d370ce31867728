// Shared definitions of the CUDA side of the fused MoE layer.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <utility>

#include "../../include/moe.h"

namespace moe {

constexpr int kWarp = 32;
// Pipeline waits inside a kernel give up after a wall-time limit (a launch
// argument: kWaitLimitNs unless moe_debug_timeouts lowered it), set an error
// in the status word and let the kernel return (no trap, no hang).
constexpr uint64_t kWaitLimitNs = 2000000000ull;
// After giving up, a role waits for its own asynchronous operations still in
// flight (TMA loads, MMAs) before the CTA frees TMEM and exits; those waits
// have their own limit, which the debug hook does not lower: the operations
// complete on their own within microseconds.
constexpr uint64_t kDrainLimitNs = 1000000000ull;

// Wait limit and start-barrier surplus for the next launches (process-wide;
// set by moe_debug_timeouts, read when a launch's arguments are filled).
uint64_t launch_wait_limit_ns();
int launch_unreachable_arrivals();

// Programmatic dependent launch: every kernel of the layer is launched with
// programmatic stream serialisation, so it may start (prologue: barrier
// init, TMEM allocation, tensor-map prefetch) while the previous kernel in
// the stream drains.  Before its first global-memory access it waits for the
// previous grid to complete and flush (griddepcontrol.wait; a no-op when the
// kernel was launched without the attribute), and it lets the next kernel
// launch early (griddepcontrol.launch_dependents).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

__device__ __forceinline__ void set_status(int32_t* status, int32_t code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
  __nv_bfloat16 v = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&v);
}

// Internal launchers (one translation unit each).
cudaError_t launch_route(const float* logits, int T, int E, int k, int n_group, int topk_group, int group_score,
                         int renormalize, float routed_scaling, int32_t* topk_ids, float* topk_weights,
                         int32_t* status, cudaStream_t stream, int* launches);

int align_num_chunks(int S);
bool align_uses_single_block(int S);
cudaError_t launch_align(const int32_t* topk_ids, int S, int E, int block_m, int P_max, int32_t* sorted_ids,
                         int32_t* expert_ids, int32_t* ntpp, int32_t* inv_pos, int32_t* ws, int32_t* status,
                         cudaStream_t stream, int* launches);

bool route_align_fusable(int T, int k, int n_group);
cudaError_t launch_route_align(const float* logits, int T, int E, int k, int n_group, int topk_group,
                               int group_score, int renormalize, float routed_scaling, int32_t* topk_ids,
                               float* topk_weights, int block_m, int P_max, int32_t* sorted_ids, int32_t* expert_ids,
                               int32_t* ntpp, int32_t* inv_pos, int32_t* status, cudaStream_t stream, int* launches);

// x_sorted[p] = x[sorted_ids[p] / k] for live rows p < ntpp, x_sorted[ntpp + t]
// = x[t] for t < min(T, n_shared_rows); with zero_pad, the other rows up to
// ntpp + n_shared_rows are set to zero.
cudaError_t launch_permute_rows(const uint16_t* x, const int32_t* sorted_ids, const int32_t* ntpp, int T, int k,
                                int d, int P_max, int n_shared_rows, uint16_t* x_sorted, int num_sms,
                                cudaStream_t stream, int* launches, bool zero_pad = false);

// Router projection on the CUDA cores: logits [T, E] fp32 = x [T, d] .
// W_g [E, d]^T (d a multiple of 8), CTAs of 8 experts x kRouterGemvMaxT
// tokens (kRouterGemvMaxT * d * 2 bytes of shared memory).
constexpr int kRouterGemvMaxT = 16;
// batches up to this many tokens take the CUDA-core product (measured: 256
// tokens 50.7 -> 23.9 us against the tensor-core path; 4096 tokens 36 -> 72 us)
constexpr int kRouterGemvTokens = 1024;
cudaError_t launch_router_gemv(const uint16_t* x, const uint16_t* w_gate, int T, int d, int E, float* logits,
                               cudaStream_t stream, int* launches);

// out = bf16(acc) over n = T * d elements (the scatter-reduce's last step).
cudaError_t launch_convert(const float* acc, int64_t n, uint16_t* out, int num_sms, cudaStream_t stream,
                           int* launches);

}  // namespace moe
