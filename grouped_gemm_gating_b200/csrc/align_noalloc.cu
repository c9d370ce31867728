// moe_align_noalloc: the align step without any caller-provided or
// library-allocated device memory beyond its inputs and outputs.
//
// For callers that cannot call cudaMalloc: runtimes that reserve all device
// memory up front and hand out none afterwards (a serving engine that has
// given the remaining HBM to its KV cache), code that runs while a stream is
// being captured into a CUDA graph (where an allocation would synchronise
// the device and break the capture), and plugins whose host framework owns
// every allocation.  Such callers cannot provide moe_align's workspace.
//
// The multi-block align path needs per-chunk expert counts; here they live
// in a file-scope static __device__ array of fixed size, which
// every GPU that loads this library holds until the process exits.
#include <cuda.h>

#include <mutex>

#include "common.cuh"

namespace moe {
void record_launches(int n);
}

namespace {

// 256 Ki int32 = 1 MiB: counts of ceil(T*k / 2048) chunks x E experts,
// i.e. ceil(T*k / 2048) * E <= 262144.
constexpr size_t kScratchInts = 262144;
static __device__ __align__(256) int32_t g_align_scratch[kScratchInts];

// In host code g_align_scratch is only a host-side stand-in for the device
// array, so its address must not be handed to a kernel.  The device address
// is looked up with cudaGetSymbolAddress, with that device current, the first
// time a device's context is seen, and cached next to that context: a new
// context on the same device (after cudaDeviceReset, say) holds the array at
// a new address, so a change of context makes the next call look it up again.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

int32_t* scratch_on_current_device(cudaError_t* err) {
  static int32_t* cache[64] = {nullptr};
  static CUcontext cache_ctx[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= 64) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  CtxGetCurrentFn get_ctx = ctx_get_current_fn();
  CUcontext ctx = nullptr;
  if (get_ctx == nullptr || get_ctx(&ctx) != CUDA_SUCCESS) {
    *err = cudaErrorInitializationError;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (ctx == nullptr || cache[dev] == nullptr || cache_ctx[dev] != ctx) {
    void* p = nullptr;
    // also makes the device's context current if no call has done so yet
    *err = cudaGetSymbolAddress(&p, g_align_scratch);
    if (*err != cudaSuccess) return nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) {
      *err = cudaErrorInitializationError;
      return nullptr;
    }
    cache[dev] = static_cast<int32_t*>(p);
    cache_ctx[dev] = ctx;
  }
  return cache[dev];
}

}  // namespace

extern "C" MOE_API moe_status moe_align_noalloc(const int32_t* topk_ids, int T, int k, int E, int block_m,
                                                int32_t* sorted_token_ids, int32_t* expert_ids,
                                                int32_t* num_tokens_post_padded, int32_t* inv_pos,
                                                int32_t* dev_status, moe_stream_t stream) {
  if (T < 0 || E < 1 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (!(block_m == 16 || block_m == 32 || block_m == 64 || block_m == 128)) return MOE_ERR_INVALID_ARG;
  if (E > MOE_MAX_EXPERTS || k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(T) * k >= (int64_t(1) << 30)) return MOE_ERR_UNSUPPORTED;
  if (!sorted_token_ids || !expert_ids || !num_tokens_post_padded) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!topk_ids || !inv_pos)) return MOE_ERR_INVALID_ARG;
  const size_t need = moe_align_workspace_size(T, k, E);
  if (need > sizeof(g_align_scratch)) return MOE_ERR_UNSUPPORTED;  // beyond the static scratch
  int32_t* ws = nullptr;
  if (need > 0) {
    cudaError_t err = cudaSuccess;
    ws = scratch_on_current_device(&err);
    if (ws == nullptr) return MOE_ERR_CUDA;
  }
  const int S = T * k;
  const int64_t P_max = moe_max_padded(T, k, E, block_m);
  int launches = 0;
  // The count kernel overwrites every count it owns, so no part of the
  // scratch has to start at zero.
  cudaError_t err = moe::launch_align(topk_ids, S, E, block_m, static_cast<int>(P_max), sorted_token_ids,
                                      expert_ids, num_tokens_post_padded, inv_pos, ws, dev_status,
                                      reinterpret_cast<cudaStream_t>(stream), &launches);
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  moe::record_launches(launches);
  return MOE_OK;
}
