// C ABI of the fused MoE layer: argument checks, workspace layout, TMA
// tensor-map encoding and the launch sequence.  See include/moe.h for the
// contract of every entry point.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>
#include <vector>

#include "../../include/moe.h"
#include "common.cuh"
#include "fused.h"
#include "gemm.h"

namespace {

thread_local int g_last_launches = 0;

// ---- stage profiling: event pairs recorded around each kernel launch ----
// Events come from a per-thread pool, so that recording (also while a stream
// is being captured into a CUDA graph) creates no event once the pool is
// primed by moe_profile_enable.
struct StageRecord {
  int stage;
  cudaEvent_t start, stop;
};
thread_local bool g_profile = false;
thread_local std::vector<StageRecord> g_records;
thread_local std::vector<cudaEvent_t> g_event_pool;
constexpr int kEventPoolPrime = 64;

// Under stream capture a plain event record only orders work inside the
// capture; the external flag makes it an event-record node of the graph, so
// the event is recorded (with its timestamp) at every replay.
cudaError_t record_event(cudaEvent_t ev, cudaStream_t stream) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return cudaErrorUnknown;
  if (cs == cudaStreamCaptureStatusActive) return cudaEventRecordWithFlags(ev, stream, cudaEventRecordExternal);
  return cudaEventRecord(ev, stream);
}

bool take_event(cudaEvent_t* ev) {
  if (!g_event_pool.empty()) {
    *ev = g_event_pool.back();
    g_event_pool.pop_back();
    return true;
  }
  return cudaEventCreate(ev) == cudaSuccess;
}

struct StageScope {
  StageRecord rec{};
  cudaStream_t stream;
  bool active;
  StageScope(int stage, cudaStream_t s) : stream(s), active(g_profile) {
    if (!active) return;
    rec.stage = stage;
    if (!take_event(&rec.start)) {
      active = false;
      return;
    }
    if (!take_event(&rec.stop)) {
      g_event_pool.push_back(rec.start);
      active = false;
      return;
    }
    if (record_event(rec.start, stream) != cudaSuccess) {
      g_event_pool.push_back(rec.start);
      g_event_pool.push_back(rec.stop);
      active = false;
    }
  }
  ~StageScope() {
    if (!active) return;
    if (record_event(rec.stop, stream) == cudaSuccess) {
      g_records.push_back(rec);
    } else {
      g_event_pool.push_back(rec.start);
      g_event_pool.push_back(rec.stop);
    }
  }
};

void release_records() {
  for (auto& r : g_records) {
    g_event_pool.push_back(r.start);
    g_event_pool.push_back(r.stop);
  }
  g_records.clear();
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int num_sms_current_device() {
  static std::atomic<int> cache[64];  // per device; concurrent first calls store the same value
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// bf16 tensor [depth, rows, K] (K innermost) as a 3-D map with 64 x box_rows
// boxes and 128-byte swizzle; zero fill out of bounds.
bool encode_3d(CUtensorMap* map, const void* base, uint64_t K, uint64_t rows, uint64_t depth, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {K, rows, depth};
  const cuuint64_t strides[2] = {K * 2, rows * K * 2};
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_2d(CUtensorMap* map, const void* base, uint64_t K, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {K, rows};
  const cuuint64_t strides[1] = {K * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// uint8 tensor [depth, rows, inner] (inner contiguous) as a 3-D map with
// box_inner x box_rows boxes, no swizzle; zero fill out of bounds.
bool encode_3d_u8(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t depth,
                  uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {inner, rows, depth};
  const cuuint64_t strides[2] = {inner, rows * inner};
  const cuuint32_t box[3] = {box_inner, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// fp8 expert weights (e4m3 values [E, rows, K] and their scale bytes
// [E, K / 32, rows]) for the fused expert kernel.
struct Fp8Weights {
  const uint8_t *w13, *s13, *w2, *s2;      // routed experts
  const uint8_t *w13s, *s13s, *w2s, *s2s;  // shared expert (n_shared == 1)
};

bool valid_block_m(int bm) { return bm == 16 || bm == 32 || bm == 64 || bm == 128; }

constexpr size_t kWsAlign = 256;
// The forward workspace starts with a fixed block of int32 counters that the
// fused expert kernel keeps at zero between calls (the last CTA of every
// launch resets them; it uses the first three as grid counters, the rest is
// reserved).  h (block_m = 128) and the fp32 accumulator follow it.
constexpr size_t kCounterInts = 16384;

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// The token-major GEMMs run on CTA pairs when the layer is wide enough for
// the K loops to dominate a tile: d_ff >= 1024 for both GEMMs (and d >= 1024
// for the gate/up GEMM, whose token rows are first copied into the
// expert-sorted order so that it can read them by TMA).  With a narrow d_ff
// the down GEMM's epilogue bounds it, blocks left unpaired only add work,
// and the copy of x outgrows what the gathered rows cost from L2.
bool uses_pair_gate_up(int block_m, int d, int F, int64_t P_total) {
  return block_m == 128 && d >= 1024 && F >= 1024 &&
         moe::gemm_pair_supported(block_m, static_cast<int>(P_total / block_m));
}

int64_t padded_total(int T, int k, int E, int bm, int n_shared) {
  const int64_t pmax = moe_max_padded(T, k, E, bm);
  if (pmax < 0) return -1;
  const int64_t shared_rows = n_shared ? (static_cast<int64_t>(T) + bm - 1) / bm * bm : 0;
  return pmax + shared_rows;
}

moe_status check_dims(int T, int d, int F, int E, int k) {
  if (T < 0 || E < 1 || k < 1 || d < 1 || F < 1) return MOE_ERR_INVALID_ARG;
  if (k > E) return MOE_ERR_INVALID_ARG;
  if (E > MOE_MAX_EXPERTS || k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
  if (d % 64 || F % 64 || d > 16384 || F > 16384) return MOE_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(T) * k >= (int64_t(1) << 30)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status finish(cudaError_t err, int launches) {
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  g_last_launches = launches;
  return MOE_OK;
}

moe_status check_route_args(int T, int E, int k, int n_group, int topk_group, moe_group_score group_score,
                            float routed_scaling) {
  if (T < 0 || E < 1 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (E > MOE_MAX_EXPERTS || k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
  if (n_group < 1 || E % n_group != 0 || topk_group < 1 || topk_group > n_group) return MOE_ERR_INVALID_ARG;
  if (static_cast<int64_t>(k) > static_cast<int64_t>(topk_group) * (E / n_group)) return MOE_ERR_INVALID_ARG;
  if (group_score != MOE_GROUP_MAX && group_score != MOE_GROUP_TOP2SUM) return MOE_ERR_INVALID_ARG;
  if (!(routed_scaling > 0.0f) || routed_scaling > 3.0e38f) return MOE_ERR_INVALID_ARG;
  if (static_cast<int64_t>(T) * k >= (int64_t(1) << 30)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status check_align_args(const int32_t* topk_ids, int T, int k, int E, int block_m,
                            const int32_t* sorted_token_ids, const int32_t* expert_ids,
                            const int32_t* num_tokens_post_padded, const int32_t* inv_pos, const void* ws,
                            size_t ws_bytes) {
  if (T < 0 || E < 1 || k < 1 || k > E || !valid_block_m(block_m)) return MOE_ERR_INVALID_ARG;
  if (E > MOE_MAX_EXPERTS || k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(T) * k >= (int64_t(1) << 30)) return MOE_ERR_UNSUPPORTED;
  if (!sorted_token_ids || !expert_ids || !num_tokens_post_padded) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!topk_ids || !inv_pos)) return MOE_ERR_INVALID_ARG;
  const size_t need = moe_align_workspace_size(T, k, E);
  if (need > 0 && (ws == nullptr || ws_bytes < need || !aligned16(ws))) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}


// Regions of the backward's workspace, each 256-byte aligned: the token rows
// and the dL/dout rows in expert-sorted order, the fp32 pre-activations,
// their gradient da (bf16), w * h, and the fp32 dx accumulator.
struct BwdLayout {
  int64_t P_total;
  size_t xs, gs, pre, da, hw, acc, total;
};

BwdLayout bwd_layout(int T, int d, int F, int E, int k, moe_act act, int n_shared) {
  BwdLayout L{};
  L.P_total = padded_total(T, k, E, 128, n_shared);
  const size_t P = static_cast<size_t>(L.P_total);
  const size_t n1 = act == MOE_ACT_SWIGLU ? 2 * static_cast<size_t>(F) : static_cast<size_t>(F);
  L.xs = 0;
  L.gs = L.xs + round_up(P * d * 2, kWsAlign);
  L.pre = L.gs + round_up(P * d * 2, kWsAlign);
  L.da = L.pre + round_up(P * n1 * 4, kWsAlign);
  L.hw = L.da + round_up(P * n1 * 2, kWsAlign);
  L.acc = L.hw + round_up(P * F * 2, kWsAlign);
  L.total = L.acc + round_up(static_cast<size_t>(T) * d * 4, kWsAlign);
  return L;
}

}  // namespace

namespace moe {
void record_launches(int n) { g_last_launches = n; }

// Set by moe_debug_timeouts; read when a launch's arguments are filled.
std::atomic<uint64_t> g_wait_limit_ns{kWaitLimitNs};
std::atomic<int> g_unreachable{0};
uint64_t launch_wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }
int launch_unreachable_arrivals() { return g_unreachable.load(std::memory_order_relaxed); }
}  // namespace moe

extern "C" {

int64_t moe_max_padded(int T, int k, int E, int block_m) {
  if (T < 0 || k < 1 || E < 1 || !valid_block_m(block_m)) return -1;
  const int64_t S = static_cast<int64_t>(T) * k;
  const int64_t p = S + static_cast<int64_t>(E) * (block_m - 1);
  return (p + block_m - 1) / block_m * block_m;
}

size_t moe_align_workspace_size(int T, int k, int E) {
  if (T < 0 || k < 1 || E < 1 || E > MOE_MAX_EXPERTS) return 0;
  const int64_t S = static_cast<int64_t>(T) * k;
  if (S >= (int64_t(1) << 30)) return 0;
  if (moe::align_uses_single_block(static_cast<int>(S))) return 0;
  return static_cast<size_t>(moe::align_num_chunks(static_cast<int>(S))) * E * sizeof(int32_t);  // per-chunk counts
}

size_t moe_workspace_size(int T, int d, int F, int E, int k, int block_m, moe_act act, int n_shared) {
  if (check_dims(T, d, F, E, k) != MOE_OK || !valid_block_m(block_m)) return 0;
  if ((act != MOE_ACT_SWIGLU && act != MOE_ACT_RELU2) || (n_shared != 0 && n_shared != 1)) return 0;
  const int64_t P = padded_total(T, k, E, block_m, n_shared);
  const size_t h = block_m == 128 ? round_up(static_cast<size_t>(P) * F * 2, kWsAlign) : 0;
  const size_t acc = round_up(static_cast<size_t>(T) * d * 4, kWsAlign);
  // permuted x for the paired gate/up GEMM
  const size_t xs = uses_pair_gate_up(block_m, d, F, P) ? round_up(static_cast<size_t>(P) * d * 2, kWsAlign) : 0;
  return kCounterInts * 4 + h + acc + xs + kWsAlign;
}

moe_status moe_route(const float* logits, int T, int E, int k, int n_group, int topk_group,
                     moe_group_score group_score, int renormalize, float routed_scaling, int32_t* topk_ids,
                     float* topk_weights, int32_t* dev_status, moe_stream_t stream) {
  moe_status st = check_route_args(T, E, k, n_group, topk_group, group_score, routed_scaling);
  if (st != MOE_OK) return st;
  if (T == 0) return finish(cudaSuccess, 0);
  if (!logits || !topk_ids || !topk_weights) return MOE_ERR_INVALID_ARG;
  int launches = 0;
  StageScope scope(0, reinterpret_cast<cudaStream_t>(stream));
  cudaError_t err = moe::launch_route(logits, T, E, k, n_group, topk_group, static_cast<int>(group_score),
                                      renormalize ? 1 : 0, routed_scaling, topk_ids, topk_weights, dev_status,
                                      reinterpret_cast<cudaStream_t>(stream), &launches);
  return finish(err, launches);
}

moe_status moe_route_align(const float* logits, int T, int E, int k, int n_group, int topk_group,
                           moe_group_score group_score, int renormalize, float routed_scaling, int block_m,
                           int32_t* topk_ids, float* topk_weights, int32_t* sorted_token_ids, int32_t* expert_ids,
                           int32_t* num_tokens_post_padded, int32_t* inv_pos, void* ws, size_t ws_bytes,
                           int32_t* dev_status, moe_stream_t stream) {
  moe_status st = check_route_args(T, E, k, n_group, topk_group, group_score, routed_scaling);
  if (st != MOE_OK) return st;
  st = check_align_args(topk_ids, T, k, E, block_m, sorted_token_ids, expert_ids, num_tokens_post_padded, inv_pos,
                        ws, ws_bytes);
  if (st != MOE_OK) return st;
  if (T > 0 && (!logits || !topk_weights)) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t P_max = moe_max_padded(T, k, E, block_m);
  int launches = 0;
  cudaError_t err = cudaSuccess;
  if (T > 0 && moe::route_align_fusable(T, k, n_group)) {
    StageScope scope(5, s);
    err = moe::launch_route_align(logits, T, E, k, n_group, topk_group, static_cast<int>(group_score),
                                  renormalize ? 1 : 0, routed_scaling, topk_ids, topk_weights, block_m,
                                  static_cast<int>(P_max), sorted_token_ids, expert_ids, num_tokens_post_padded,
                                  inv_pos, dev_status, s, &launches);
    return finish(err, launches);
  }
  if (T > 0) {
    StageScope scope(0, s);
    err = moe::launch_route(logits, T, E, k, n_group, topk_group, static_cast<int>(group_score), renormalize ? 1 : 0,
                            routed_scaling, topk_ids, topk_weights, dev_status, s, &launches);
  }
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  {
    StageScope scope(1, s);
    err = moe::launch_align(topk_ids, T * k, E, block_m, static_cast<int>(P_max), sorted_token_ids, expert_ids,
                            num_tokens_post_padded, inv_pos, static_cast<int32_t*>(ws), dev_status, s, &launches);
  }
  return finish(err, launches);
}

moe_status moe_align(const int32_t* topk_ids, int T, int k, int E, int block_m, int32_t* sorted_token_ids,
                     int32_t* expert_ids, int32_t* num_tokens_post_padded, int32_t* inv_pos, void* ws,
                     size_t ws_bytes, int32_t* dev_status, moe_stream_t stream) {
  moe_status st = check_align_args(topk_ids, T, k, E, block_m, sorted_token_ids, expert_ids, num_tokens_post_padded,
                                   inv_pos, ws, ws_bytes);
  if (st != MOE_OK) return st;
  const int S = T * k;
  const int64_t P_max = moe_max_padded(T, k, E, block_m);
  int launches = 0;
  StageScope scope(1, reinterpret_cast<cudaStream_t>(stream));
  cudaError_t err = moe::launch_align(topk_ids, S, E, block_m, static_cast<int>(P_max), sorted_token_ids,
                                      expert_ids, num_tokens_post_padded, inv_pos, static_cast<int32_t*>(ws),
                                      dev_status, reinterpret_cast<cudaStream_t>(stream), &launches);
  return finish(err, launches);
}

}  // extern "C"

namespace {

// The forward after its argument checks.  route != nullptr: the fused kernel
// also routes and aligns (the caller checked fused_routing_supported), and
// topk_weights / sorted_token_ids / expert_ids / num_tokens_post_padded are
// written by it instead of read.
moe_status forward_impl(const uint16_t* x, int T, int d, const uint16_t* w13, const uint16_t* w2, int E, int F,
                        const uint16_t* w13_shared, const uint16_t* w2_shared, int n_shared,
                        const float* topk_weights, int k, const int32_t* sorted_token_ids,
                        const int32_t* expert_ids, const int32_t* num_tokens_post_padded, int block_m, moe_act act,
                        uint16_t* out, void* ws, int32_t* dev_status, cudaStream_t s, int* launches_io,
                        const moe::FusedRoute* route, const Fp8Weights* fp8 = nullptr) {
  const int bm = block_m;
  const int64_t P_max = moe_max_padded(T, k, E, bm);
  const int64_t P_total = padded_total(T, k, E, bm, n_shared);
  const int n_shared_blocks = n_shared ? (T + bm - 1) / bm : 0;
  const int max_routed_blocks = static_cast<int>(P_max / bm);
  uint8_t* wsb = reinterpret_cast<uint8_t*>(round_up(reinterpret_cast<uintptr_t>(ws), kWsAlign));
  int32_t* counters = reinterpret_cast<int32_t*>(wsb);
  // workspace: counters, then h (block_m = 128 only), then the fp32 [T, d] accumulator
  uint16_t* h = reinterpret_cast<uint16_t*>(wsb + kCounterInts * 4);
  const size_t h_bytes = bm == 128 ? round_up(static_cast<size_t>(P_total) * F * 2, kWsAlign) : 0;
  float* y = reinterpret_cast<float*>(wsb + kCounterInts * 4 + h_bytes);
  uint16_t* x_sorted = reinterpret_cast<uint16_t*>(wsb + kCounterInts * 4 + h_bytes +
                                                   round_up(static_cast<size_t>(T) * d * 4, kWsAlign));
  const int n1 = act == MOE_ACT_SWIGLU ? 2 * F : F;
  const int num_sms = num_sms_current_device();
  if (num_sms <= 0) return MOE_ERR_CUDA;
  int& launches = *launches_io;
  const int total_blocks_max = static_cast<int>(P_total / bm);

  if (moe::fused_expert_supported(bm)) {
    // small token blocks: both GEMMs and the scatter-reduce in one persistent
    // kernel that accumulates into the fp32 y region; its three grid
    // counters are zero on entry and are returned to zero by its last CTA
    moe::FusedArgs fa;
    std::memset(&fa, 0, sizeof(fa));
    // gate/up tiles: 64 gate rows + 64 up rows (SwiGLU) or 128 fc1 rows,
    // loaded in boxes of the kernel's box height; W2 tiles: 128 d rows
    const uint32_t box13 = act == MOE_ACT_SWIGLU ? moe::kFusedBoxRowsGated : moe::kFusedBoxRowsRelu2;
    const uint32_t box2 = moe::kFusedBoxRowsW2;
    if (fp8 != nullptr) {
      // e4m3 weights in boxes of 64 K bytes x 128 rows; scale bytes in boxes
      // of 128 rows x 2 K blocks
      if (!encode_3d_u8(&fa.tm_w13, fp8->w13, d, n1, E, 64, 128) || !encode_3d_u8(&fa.tm_w2, fp8->w2, F, d, E, 64, 128) ||
          !encode_3d_u8(&fa.tm_s13, fp8->s13, n1, d / 32, E, 128, 2) ||
          !encode_3d_u8(&fa.tm_s2, fp8->s2, d, F / 32, E, 128, 2))
        return MOE_ERR_CUDA;
      if (n_shared) {
        if (!encode_3d_u8(&fa.tm_w13s, fp8->w13s, d, n1, 1, 64, 128) ||
            !encode_3d_u8(&fa.tm_w2s, fp8->w2s, F, d, 1, 64, 128) ||
            !encode_3d_u8(&fa.tm_s13s, fp8->s13s, n1, d / 32, 1, 128, 2) ||
            !encode_3d_u8(&fa.tm_s2s, fp8->s2s, d, F / 32, 1, 128, 2))
          return MOE_ERR_CUDA;
      } else {
        fa.tm_w13s = fa.tm_w13;
        fa.tm_w2s = fa.tm_w2;
        fa.tm_s13s = fa.tm_s13;
        fa.tm_s2s = fa.tm_s2;
      }
    } else {
      if (!encode_3d(&fa.tm_w13, w13, d, n1, E, box13) || !encode_3d(&fa.tm_w2, w2, F, d, E, box2))
        return MOE_ERR_CUDA;
      if (n_shared) {
        if (!encode_3d(&fa.tm_w13s, w13_shared, d, n1, 1, box13) || !encode_3d(&fa.tm_w2s, w2_shared, F, d, 1, box2))
          return MOE_ERR_CUDA;
      } else {
        fa.tm_w13s = fa.tm_w13;
        fa.tm_w2s = fa.tm_w2;
      }
    }
    fa.x = x;
    fa.acc = y;
    fa.out = out;
    fa.sorted_ids = sorted_token_ids;
    fa.expert_ids = expert_ids;
    fa.ntpp = num_tokens_post_padded;
    fa.topk_w = topk_weights;
    fa.sync = counters;
    fa.status = dev_status;
    fa.wait_ns = moe::launch_wait_limit_ns();
    fa.start_surplus = moe::launch_unreachable_arrivals();
    fa.T = T;
    fa.k = k;
    fa.S = T * k;
    fa.E = E;
    fa.d = d;
    fa.F = F;
    fa.block_m = bm;
    fa.max_routed_blocks = max_routed_blocks;
    fa.n_shared_blocks = n_shared_blocks;
    const int epi = act == MOE_ACT_SWIGLU ? moe::kEpiSwiGLU : moe::kEpiRelu2;
    const int64_t tiles = moe::fused_expert_max_tiles(epi, total_blocks_max, F);
    const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
    if (route != nullptr) fa.route = *route;
    cudaError_t err;
    {
      StageScope scope(6, s);
      err = moe::launch_fused_expert(epi, bm, route != nullptr, fa, grid < 1 ? 1 : grid, s, fp8 != nullptr);
    }
    if (err != cudaSuccess) return MOE_ERR_CUDA;
    ++launches;
    return finish(err, launches);
  }

  // gate/up (or fc1) GEMM with the activation epilogue: h [P_total, F]
  moe::GemmArgs a1;
  std::memset(&a1, 0, sizeof(a1));
  const int epi1 = act == MOE_ACT_SWIGLU ? moe::kEpiSwiGLU : moe::kEpiRelu2;
  const bool pair1 = uses_pair_gate_up(bm, d, F, P_total);
  const uint32_t box1 = pair1 ? 128u : static_cast<uint32_t>(moe::gemm_box_rows(epi1));
  if (!encode_3d(&a1.tm_w, w13, d, n1, E, box1)) return MOE_ERR_CUDA;
  if (n_shared) {
    if (!encode_3d(&a1.tm_ws, w13_shared, d, n1, 1, box1)) return MOE_ERR_CUDA;
  } else {
    a1.tm_ws = a1.tm_w;
  }
  if (pair1) {
    // token rows by TMA from x permuted into the expert-sorted order
    if (!encode_2d(&a1.tm_x, x_sorted, d, static_cast<uint64_t>(P_total), 128)) return MOE_ERR_CUDA;
  } else {
    a1.tm_x = a1.tm_w;  // unused: the single-CTA kernel gathers rows with cp.async
  }
  a1.x = x;
  a1.sorted_ids = sorted_token_ids;
  a1.expert_ids = expert_ids;
  a1.ntpp = num_tokens_post_padded;
  a1.topk_w = topk_weights;
  a1.out = h;
  a1.acc = y;  // zeroed on the side for the down GEMM
  a1.acc_elems = static_cast<int64_t>(T) * d;
  a1.status = dev_status;
  a1.wait_ns = moe::launch_wait_limit_ns();
  a1.tfull_surplus = moe::launch_unreachable_arrivals();
  a1.T = T;
  a1.k = k;
  a1.S = T * k;
  a1.E = E;
  a1.K = d;
  a1.n_out = F;
  a1.up_row_offset = F;
  a1.block_m = bm;
  a1.max_routed_blocks = max_routed_blocks;
  a1.n_shared_blocks = n_shared_blocks;
  int64_t tiles = moe::gemm_max_tiles(epi1, max_routed_blocks, n_shared_blocks, F);
  int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
  if (grid < 1) grid = 1;
  cudaError_t err;
  {
    StageScope scope(2, s);
    if (pair1) {
      {
        StageScope pscope(7, s);
        err = moe::launch_permute_rows(x, sorted_token_ids, num_tokens_post_padded, T, k, d, static_cast<int>(P_max),
                                       n_shared_blocks * bm, x_sorted, num_sms, s, &launches);
      }
      if (err == cudaSuccess) err = moe::launch_grouped_gemm_pair(epi1, a1, num_sms & ~1, s);
    } else if (moe::gemm_wide_supported(epi1, bm, total_blocks_max)) {
      err = moe::launch_grouped_gemm_wide(epi1, a1, grid, s);
    } else {
      err = moe::launch_grouped_gemm(epi1, a1, grid, s);
    }
  }
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  ++launches;

  // down GEMM whose epilogue adds topk_weight * row into acc [T, d] fp32
  moe::GemmArgs a2;
  std::memset(&a2, 0, sizeof(a2));
  // CTA pairs share each 256-row W2 tile (128 rows per CTA).  Worth it when
  // the K loop is long (d_ff >= 1024); with a short one the epilogue's
  // reductions bound the kernel and unpaired blocks would only add work.
  const bool pair2 = F >= 1024 && moe::gemm_pair_supported(bm, total_blocks_max);
  const uint32_t box2 = pair2 ? 128u : static_cast<uint32_t>(moe::gemm_box_rows(moe::kEpiScale));
  if (!encode_3d(&a2.tm_w, w2, F, d, E, box2)) return MOE_ERR_CUDA;
  if (n_shared) {
    if (!encode_3d(&a2.tm_ws, w2_shared, F, d, 1, box2)) return MOE_ERR_CUDA;
  } else {
    a2.tm_ws = a2.tm_w;
  }
  if (!encode_2d(&a2.tm_x, h, F, static_cast<uint64_t>(P_total), static_cast<uint32_t>(bm))) return MOE_ERR_CUDA;
  a2.x = nullptr;
  a2.sorted_ids = sorted_token_ids;
  a2.expert_ids = expert_ids;
  a2.ntpp = num_tokens_post_padded;
  a2.topk_w = topk_weights;
  a2.out = nullptr;
  a2.acc = y;
  a2.acc_elems = static_cast<int64_t>(T) * d;
  a2.status = dev_status;
  a2.wait_ns = moe::launch_wait_limit_ns();
  a2.tfull_surplus = moe::launch_unreachable_arrivals();
  a2.T = T;
  a2.k = k;
  a2.S = T * k;
  a2.E = E;
  a2.K = F;
  a2.n_out = d;
  a2.up_row_offset = 0;
  a2.block_m = bm;
  a2.max_routed_blocks = max_routed_blocks;
  a2.n_shared_blocks = n_shared_blocks;
  {
    // column passes: keep each pass's slice of the accumulator within ~48 MB of L2
    const int64_t acc_bytes = static_cast<int64_t>(T) * d * 4;
    const int64_t budget = int64_t(48) << 20;
    const int n_wt = (d + 255) / 256;
    const int passes = static_cast<int>((acc_bytes + budget - 1) / budget);
    a2.pass_cols = passes <= 1 ? 0 : (n_wt + passes - 1) / passes;
  }
  tiles = moe::gemm_max_tiles(moe::kEpiScale, max_routed_blocks, n_shared_blocks, d);
  grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
  if (grid < 1) grid = 1;
  {
    StageScope scope(3, s);
    if (pair2)
      err = moe::launch_grouped_gemm_pair(moe::kEpiScale, a2, num_sms & ~1, s);
    else
      err = moe::launch_grouped_gemm(moe::kEpiScale, a2, grid, s);
  }
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  ++launches;

  {
    StageScope scope(4, s);
    err = moe::launch_convert(y, static_cast<int64_t>(T) * d, out, num_sms, s, &launches);
  }
  return finish(err, launches);
}

}  // namespace

namespace {

moe_status forward_checked(const uint16_t* x, int T, int d, const uint16_t* w13, const uint16_t* w2, int E, int F,
                       const uint16_t* w13_shared, const uint16_t* w2_shared, int n_shared,
                       const float* topk_weights, int k, const int32_t* sorted_token_ids,
                       const int32_t* expert_ids, const int32_t* num_tokens_post_padded, const int32_t* inv_pos,
                       int block_m, moe_act act, uint16_t* out, void* ws, size_t ws_bytes, int32_t* dev_status,
                       moe_stream_t stream, const Fp8Weights* fp8) {
  moe_status st = check_dims(T, d, F, E, k);
  if (st != MOE_OK) return st;
  if (!valid_block_m(block_m)) return MOE_ERR_UNSUPPORTED;
  if (act != MOE_ACT_SWIGLU && act != MOE_ACT_RELU2) return MOE_ERR_INVALID_ARG;
  if (n_shared != 0 && n_shared != 1) return MOE_ERR_UNSUPPORTED;
  if (n_shared && (!w13_shared || !w2_shared)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return finish(cudaSuccess, 0);
  if (!x || !w13 || !w2 || !topk_weights || !sorted_token_ids || !expert_ids || !num_tokens_post_padded || !out)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w13) || !aligned16(w2) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  if (n_shared && (!aligned16(w13_shared) || !aligned16(w2_shared))) return MOE_ERR_INVALID_ARG;
  if (fp8 != nullptr) {
    if (!moe::fused_expert_supported(block_m)) return MOE_ERR_UNSUPPORTED;  // block_m <= 64 only
    if (!fp8->s13 || !fp8->s2 || !aligned16(fp8->s13) || !aligned16(fp8->s2)) return MOE_ERR_INVALID_ARG;
    if (n_shared && (!fp8->s13s || !fp8->s2s || !aligned16(fp8->s13s) || !aligned16(fp8->s2s)))
      return MOE_ERR_INVALID_ARG;
  }
  const size_t need = moe_workspace_size(T, d, F, E, k, block_m, act, n_shared);
  if (ws == nullptr || ws_bytes < need) return MOE_ERR_WORKSPACE;

  int launches = 0;
  return forward_impl(x, T, d, w13, w2, E, F, w13_shared, w2_shared, n_shared, topk_weights, k, sorted_token_ids,
                      expert_ids, num_tokens_post_padded, block_m, act, out, ws, dev_status,
                      reinterpret_cast<cudaStream_t>(stream), &launches, nullptr, fp8);
}

moe_status layer_checked(const float* logits, int T, int E, int k, int n_group, int topk_group,
                     moe_group_score group_score, int renormalize, float routed_scaling, const uint16_t* x, int d,
                     const uint16_t* w13, const uint16_t* w2, int F, const uint16_t* w13_shared,
                     const uint16_t* w2_shared, int n_shared, int block_m, moe_act act, int32_t* topk_ids,
                     float* topk_weights, int32_t* sorted_token_ids, int32_t* expert_ids,
                     int32_t* num_tokens_post_padded, int32_t* inv_pos, uint16_t* out, void* ws, size_t ws_bytes,
                     int32_t* dev_status, moe_stream_t stream, const Fp8Weights* fp8) {
  moe_status st = check_route_args(T, E, k, n_group, topk_group, group_score, routed_scaling);
  if (st != MOE_OK) return st;
  st = check_dims(T, d, F, E, k);
  if (st != MOE_OK) return st;
  if (!valid_block_m(block_m)) return MOE_ERR_UNSUPPORTED;
  if (act != MOE_ACT_SWIGLU && act != MOE_ACT_RELU2) return MOE_ERR_INVALID_ARG;
  if (n_shared != 0 && n_shared != 1) return MOE_ERR_UNSUPPORTED;
  if (n_shared && (!w13_shared || !w2_shared)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return finish(cudaSuccess, 0);
  if (!logits || !x || !w13 || !w2 || !topk_ids || !topk_weights || !sorted_token_ids || !expert_ids ||
      !num_tokens_post_padded || !inv_pos || !out)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w13) || !aligned16(w2) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  if (n_shared && (!aligned16(w13_shared) || !aligned16(w2_shared))) return MOE_ERR_INVALID_ARG;
  if (fp8 != nullptr) {
    if (!moe::fused_expert_supported(block_m)) return MOE_ERR_UNSUPPORTED;  // block_m <= 64 only
    if (!fp8->s13 || !fp8->s2 || !aligned16(fp8->s13) || !aligned16(fp8->s2)) return MOE_ERR_INVALID_ARG;
    if (n_shared && (!fp8->s13s || !fp8->s2s || !aligned16(fp8->s13s) || !aligned16(fp8->s2s)))
      return MOE_ERR_INVALID_ARG;
  }
  const size_t need = moe_workspace_size(T, d, F, E, k, block_m, act, n_shared);
  if (ws == nullptr || ws_bytes < need) return MOE_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int launches = 0;
  if (moe::fused_expert_supported(block_m) && moe::fused_routing_supported(T, k, E, n_group, block_m)) {
    moe::FusedRoute r;
    r.logits = logits;
    r.n_group = n_group;
    r.topk_group = topk_group;
    r.group_score = static_cast<int>(group_score);
    r.renormalize = renormalize ? 1 : 0;
    r.routed_scaling = routed_scaling;
    r.topk_ids = topk_ids;
    r.topk_w = topk_weights;
    r.sorted_ids = sorted_token_ids;
    r.expert_ids = expert_ids;
    r.ntpp = num_tokens_post_padded;
    r.inv_pos = inv_pos;
    r.P_max = static_cast<int>(moe_max_padded(T, k, E, block_m));
    return forward_impl(x, T, d, w13, w2, E, F, w13_shared, w2_shared, n_shared, topk_weights, k, sorted_token_ids,
                        expert_ids, num_tokens_post_padded, block_m, act, out, ws, dev_status, s, &launches, &r, fp8);
  }
  // separate launches: routing and align (fused when the batch is small),
  // then the forward; the align scratch borrows the forward's accumulator
  // region, which the forward only touches after the align has finished
  const int P_max = static_cast<int>(moe_max_padded(T, k, E, block_m));
  cudaError_t err;
  if (moe::route_align_fusable(T, k, n_group)) {
    StageScope scope(5, s);
    err = moe::launch_route_align(logits, T, E, k, n_group, topk_group, static_cast<int>(group_score),
                                  renormalize ? 1 : 0, routed_scaling, topk_ids, topk_weights, block_m, P_max,
                                  sorted_token_ids, expert_ids, num_tokens_post_padded, inv_pos, dev_status, s,
                                  &launches);
  } else {
    {
      StageScope scope(0, s);
      err = moe::launch_route(logits, T, E, k, n_group, topk_group, static_cast<int>(group_score),
                              renormalize ? 1 : 0, routed_scaling, topk_ids, topk_weights, dev_status, s, &launches);
    }
    if (err != cudaSuccess) return MOE_ERR_CUDA;
    const size_t align_need = moe_align_workspace_size(T, k, E);
    uint8_t* wsb = reinterpret_cast<uint8_t*>(round_up(reinterpret_cast<uintptr_t>(ws), kWsAlign));
    const size_t acc_off = need - kWsAlign - round_up(static_cast<size_t>(T) * d * 4, kWsAlign);
    if (align_need > round_up(static_cast<size_t>(T) * d * 4, kWsAlign)) return MOE_ERR_WORKSPACE;
    StageScope scope(1, s);
    err = moe::launch_align(topk_ids, T * k, E, block_m, P_max, sorted_token_ids, expert_ids,
                            num_tokens_post_padded, inv_pos, reinterpret_cast<int32_t*>(wsb + acc_off), dev_status, s,
                            &launches);
  }
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  return forward_impl(x, T, d, w13, w2, E, F, w13_shared, w2_shared, n_shared, topk_weights, k, sorted_token_ids,
                      expert_ids, num_tokens_post_padded, block_m, act, out, ws, dev_status, s, &launches, nullptr, fp8);
}

}  // namespace

extern "C" {

moe_status moe_router(const uint16_t* x, int T, int d, const uint16_t* w_gate, int E, int k, int n_group,
                      int topk_group, moe_group_score group_score, int renormalize, float routed_scaling,
                      float* logits, int32_t* topk_ids, float* topk_weights, int32_t* dev_status,
                      moe_stream_t stream) {
  moe_status st = check_route_args(T, E, k, n_group, topk_group, group_score, routed_scaling);
  if (st != MOE_OK) return st;
  if (d < 64 || d % 64 != 0) return MOE_ERR_UNSUPPORTED;
  if (E > moe::kRouterMaxE || k > moe::kRouterMaxK) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return finish(cudaSuccess, 0);
  if (!x || !w_gate || !logits || !topk_ids || !topk_weights) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_gate) || (reinterpret_cast<uintptr_t>(logits) & 3u) != 0)
    return MOE_ERR_INVALID_ARG;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int launches = 0;
  if (T <= moe::kRouterGemvTokens && static_cast<int64_t>(moe::kRouterGemvMaxT) * d * 2 <= 160 * 1024) {
    // up to a thousand tokens: the product spread over (E / 8) x (T / 16)
    // CTAs on the CUDA cores (one tensor-core tile per 128 tokens would
    // leave most SMs idle); then the routing kernel gates
    cudaError_t err;
    {
      StageScope scope(8, s);
      err = moe::launch_router_gemv(x, w_gate, T, d, E, logits, s, &launches);
    }
    if (err == cudaSuccess) {
      StageScope scope(0, s);
      err = moe::launch_route(logits, T, E, k, n_group, topk_group, static_cast<int>(group_score),
                              renormalize ? 1 : 0, routed_scaling, topk_ids, topk_weights, dev_status, s, &launches);
    }
    return finish(err, launches);
  }
  const int num_sms = num_sms_current_device();
  if (num_sms <= 0) return MOE_ERR_CUDA;
  moe::GemmArgs a;
  std::memset(&a, 0, sizeof(a));
  // W_g as the single weight matrix {K = d, rows = E, 1} with 256-row boxes
  // (rows past E read as zeros); x rows by 2-D TMA, 128 tokens per block
  if (!encode_3d(&a.tm_ws, w_gate, d, static_cast<uint64_t>(E), 1, moe::kRouterMaxE)) return MOE_ERR_CUDA;
  a.tm_w = a.tm_ws;
  if (!encode_2d(&a.tm_x, x, d, static_cast<uint64_t>(T), 128)) return MOE_ERR_CUDA;
  a.status = dev_status;
  a.wait_ns = moe::launch_wait_limit_ns();
  a.tfull_surplus = moe::launch_unreachable_arrivals();
  a.T = T;
  a.k = k;
  a.S = T * k;
  a.E = E;
  a.K = d;
  a.n_out = E;
  a.block_m = 128;
  a.max_routed_blocks = 0;
  a.n_shared_blocks = (T + 127) / 128;
  a.logits = logits;
  const int grid = a.n_shared_blocks < num_sms ? a.n_shared_blocks : num_sms;
  cudaError_t err;
  {
    StageScope scope(8, s);
    err = moe::launch_grouped_gemm(moe::kEpiRouter, a, grid, s);
  }
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  ++launches;
  // the routing kernel gates the written logits, a warp per token (gating
  // in the GEMM's epilogue, a thread per token, took 59.6 us on 16384
  // tokens x 128 experts)
  {
    StageScope scope(0, s);
    err = moe::launch_route(logits, T, E, k, n_group, topk_group, static_cast<int>(group_score),
                            renormalize ? 1 : 0, routed_scaling, topk_ids, topk_weights, dev_status, s, &launches);
  }
  return finish(err, launches);
}


moe_status moe_forward(const uint16_t* x, int T, int d, const uint16_t* w13, const uint16_t* w2, int E, int F,
                       const uint16_t* w13_shared, const uint16_t* w2_shared, int n_shared,
                       const float* topk_weights, int k, const int32_t* sorted_token_ids,
                       const int32_t* expert_ids, const int32_t* num_tokens_post_padded, const int32_t* inv_pos,
                       int block_m, moe_act act, uint16_t* out, void* ws, size_t ws_bytes, int32_t* dev_status,
                       moe_stream_t stream) {
  return forward_checked(x, T, d, w13, w2, E, F, w13_shared, w2_shared, n_shared, topk_weights, k, sorted_token_ids,
                         expert_ids, num_tokens_post_padded, inv_pos, block_m, act, out, ws, ws_bytes, dev_status,
                         stream, nullptr);
}

moe_status moe_forward_fp8(const uint16_t* x, int T, int d, const uint8_t* w13_q, const uint8_t* w13_scales,
                           const uint8_t* w2_q, const uint8_t* w2_scales, int E, int F, const uint8_t* w13s_q,
                           const uint8_t* w13s_scales, const uint8_t* w2s_q, const uint8_t* w2s_scales, int n_shared,
                           const float* topk_weights, int k, const int32_t* sorted_token_ids,
                           const int32_t* expert_ids, const int32_t* num_tokens_post_padded, const int32_t* inv_pos,
                           int block_m, moe_act act, uint16_t* out, void* ws, size_t ws_bytes, int32_t* dev_status,
                           moe_stream_t stream) {
  const Fp8Weights f{w13_q, w13_scales, w2_q, w2_scales, w13s_q, w13s_scales, w2s_q, w2s_scales};
  return forward_checked(x, T, d, reinterpret_cast<const uint16_t*>(w13_q), reinterpret_cast<const uint16_t*>(w2_q),
                         E, F, reinterpret_cast<const uint16_t*>(w13s_q), reinterpret_cast<const uint16_t*>(w2s_q),
                         n_shared, topk_weights, k, sorted_token_ids, expert_ids, num_tokens_post_padded, inv_pos,
                         block_m, act, out, ws, ws_bytes, dev_status, stream, &f);
}

moe_status moe_layer(const float* logits, int T, int E, int k, int n_group, int topk_group,
                     moe_group_score group_score, int renormalize, float routed_scaling, const uint16_t* x, int d,
                     const uint16_t* w13, const uint16_t* w2, int F, const uint16_t* w13_shared,
                     const uint16_t* w2_shared, int n_shared, int block_m, moe_act act, int32_t* topk_ids,
                     float* topk_weights, int32_t* sorted_token_ids, int32_t* expert_ids,
                     int32_t* num_tokens_post_padded, int32_t* inv_pos, uint16_t* out, void* ws, size_t ws_bytes,
                     int32_t* dev_status, moe_stream_t stream) {
  return layer_checked(logits, T, E, k, n_group, topk_group, group_score, renormalize, routed_scaling, x, d, w13, w2,
                       F, w13_shared, w2_shared, n_shared, block_m, act, topk_ids, topk_weights, sorted_token_ids,
                       expert_ids, num_tokens_post_padded, inv_pos, out, ws, ws_bytes, dev_status, stream, nullptr);
}

moe_status moe_layer_fp8(const float* logits, int T, int E, int k, int n_group, int topk_group,
                         moe_group_score group_score, int renormalize, float routed_scaling, const uint16_t* x, int d,
                         const uint8_t* w13_q, const uint8_t* w13_scales, const uint8_t* w2_q,
                         const uint8_t* w2_scales, int F, const uint8_t* w13s_q, const uint8_t* w13s_scales,
                         const uint8_t* w2s_q, const uint8_t* w2s_scales, int n_shared, int block_m, moe_act act,
                         int32_t* topk_ids, float* topk_weights, int32_t* sorted_token_ids, int32_t* expert_ids,
                         int32_t* num_tokens_post_padded, int32_t* inv_pos, uint16_t* out, void* ws,
                         size_t ws_bytes, int32_t* dev_status, moe_stream_t stream) {
  const Fp8Weights f{w13_q, w13_scales, w2_q, w2_scales, w13s_q, w13s_scales, w2s_q, w2s_scales};
  return layer_checked(logits, T, E, k, n_group, topk_group, group_score, renormalize, routed_scaling, x, d,
                       reinterpret_cast<const uint16_t*>(w13_q), reinterpret_cast<const uint16_t*>(w2_q), F,
                       reinterpret_cast<const uint16_t*>(w13s_q), reinterpret_cast<const uint16_t*>(w2s_q), n_shared,
                       block_m, act, topk_ids, topk_weights, sorted_token_ids, expert_ids, num_tokens_post_padded,
                       inv_pos, out, ws, ws_bytes, dev_status, stream, &f);
}

size_t moe_backward_workspace_size(int T, int d, int F, int E, int k, moe_act act, int n_shared) {
  if (check_dims(T, d, F, E, k) != MOE_OK) return 0;
  if ((act != MOE_ACT_SWIGLU && act != MOE_ACT_RELU2) || (n_shared != 0 && n_shared != 1)) return 0;
  return bwd_layout(T, d, F, E, k, act, n_shared).total + kWsAlign;
}

moe_status moe_backward(const uint16_t* x, int T, int d, const uint16_t* w13, const uint16_t* w2, int E, int F,
                        const uint16_t* w13_shared, const uint16_t* w2_shared, int n_shared,
                        const float* topk_weights, int k, const int32_t* sorted_token_ids,
                        const int32_t* expert_ids, const int32_t* num_tokens_post_padded, moe_act act,
                        const uint16_t* dout, uint16_t* dx, uint16_t* dw13, uint16_t* dw2, uint16_t* dw13_shared,
                        uint16_t* dw2_shared, float* dtopk_weights, void* ws, size_t ws_bytes, int32_t* dev_status,
                        moe_stream_t stream) {
  moe_status st = check_dims(T, d, F, E, k);
  if (st != MOE_OK) return st;
  if (act != MOE_ACT_SWIGLU && act != MOE_ACT_RELU2) return MOE_ERR_INVALID_ARG;
  if (n_shared != 0 && n_shared != 1) return MOE_ERR_UNSUPPORTED;
  if (n_shared && (!w13_shared || !w2_shared || !dw13_shared || !dw2_shared)) return MOE_ERR_INVALID_ARG;
  if (!w13 || !w2 || !dw13 || !dw2) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w13) || !aligned16(w2) || !aligned16(dw13) || !aligned16(dw2)) return MOE_ERR_INVALID_ARG;
  if (n_shared && (!aligned16(w13_shared) || !aligned16(w2_shared) || !aligned16(dw13_shared) ||
                   !aligned16(dw2_shared)))
    return MOE_ERR_INVALID_ARG;
  if (T > 0) {
    if (!x || !topk_weights || !sorted_token_ids || !expert_ids || !num_tokens_post_padded || !dout || !dx)
      return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(dout) || !aligned16(dx)) return MOE_ERR_INVALID_ARG;
    if (dtopk_weights && !aligned16(dtopk_weights)) return MOE_ERR_INVALID_ARG;
  }
  const size_t need = moe_backward_workspace_size(T, d, F, E, k, act, n_shared);
  if (ws == nullptr || ws_bytes < need) return MOE_ERR_WORKSPACE;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int num_sms = num_sms_current_device();
  if (num_sms <= 0) return MOE_ERR_CUDA;
  const int bm = 128;
  const int n1 = act == MOE_ACT_SWIGLU ? 2 * F : F;
  const int64_t P_max = moe_max_padded(T, k, E, bm);
  const BwdLayout L = bwd_layout(T, d, F, E, k, act, n_shared);
  const int n_shared_blocks = n_shared ? (T + bm - 1) / bm : 0;
  const int max_routed_blocks = static_cast<int>(P_max / bm);
  uint8_t* wsb = reinterpret_cast<uint8_t*>(round_up(reinterpret_cast<uintptr_t>(ws), kWsAlign));
  uint16_t* xs = reinterpret_cast<uint16_t*>(wsb + L.xs);
  uint16_t* gs = reinterpret_cast<uint16_t*>(wsb + L.gs);
  float* pre = reinterpret_cast<float*>(wsb + L.pre);
  uint16_t* da = reinterpret_cast<uint16_t*>(wsb + L.da);
  uint16_t* hw = reinterpret_cast<uint16_t*>(wsb + L.hw);
  float* acc = reinterpret_cast<float*>(wsb + L.acc);
  const uint64_t wait_ns = moe::launch_wait_limit_ns();
  const int surplus = moe::launch_unreachable_arrivals();
  int launches = 0;
  cudaError_t err = cudaSuccess;
  auto grid_for = [&](int64_t tiles) { return static_cast<int>(tiles < 1 ? 1 : (tiles < num_sms ? tiles : num_sms)); };

  if (T == 0) {
    // no rows: every weight gradient is zero
    const size_t n13 = static_cast<size_t>(E) * n1 * d * 2, n2 = static_cast<size_t>(E) * d * F * 2;
    if (cudaMemsetAsync(dw13, 0, n13, s) != cudaSuccess || cudaMemsetAsync(dw2, 0, n2, s) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (n_shared && (cudaMemsetAsync(dw13_shared, 0, n13 / E, s) != cudaSuccess ||
                     cudaMemsetAsync(dw2_shared, 0, n2 / E, s) != cudaSuccess))
      return MOE_ERR_CUDA;
    return finish(cudaSuccess, 0);
  }

  // 1. token rows and dL/dout rows in the expert-sorted order, padding rows zero
  {
    StageScope scope(7, s);
    err = moe::launch_permute_rows(x, sorted_token_ids, num_tokens_post_padded, T, k, d, static_cast<int>(P_max),
                                   n_shared_blocks * bm, xs, num_sms, s, &launches, true);
    if (err == cudaSuccess)
      err = moe::launch_permute_rows(dout, sorted_token_ids, num_tokens_post_padded, T, k, d,
                                     static_cast<int>(P_max), n_shared_blocks * bm, gs, num_sms, s, &launches, true);
  }
  if (err != cudaSuccess) return MOE_ERR_CUDA;

  auto base_args = [&](moe::GemmArgs& a) {
    std::memset(&a, 0, sizeof(a));
    a.sorted_ids = sorted_token_ids;
    a.expert_ids = expert_ids;
    a.ntpp = num_tokens_post_padded;
    a.topk_w = topk_weights;
    a.status = dev_status;
    a.wait_ns = wait_ns;
    a.tfull_surplus = surplus;
    a.T = T;
    a.k = k;
    a.S = T * k;
    a.E = E;
    a.block_m = bm;
    a.max_routed_blocks = max_routed_blocks;
    a.n_shared_blocks = n_shared_blocks;
  };

  // 2. gate/up (fc1) pre-activations recomputed from the sorted token rows;
  //    a spare warp zeroes the dx accumulator and dL/d topk_weights
  {
    moe::GemmArgs a;
    base_args(a);
    const int epi = act == MOE_ACT_SWIGLU ? moe::kEpiPreSwiGLU : moe::kEpiPreRelu2;
    const uint32_t box = static_cast<uint32_t>(moe::gemm_box_rows(epi));
    if (!encode_3d(&a.tm_w, w13, d, n1, E, box)) return MOE_ERR_CUDA;
    if (n_shared) {
      if (!encode_3d(&a.tm_ws, w13_shared, d, n1, 1, box)) return MOE_ERR_CUDA;
    } else {
      a.tm_ws = a.tm_w;
    }
    if (!encode_2d(&a.tm_x, xs, d, static_cast<uint64_t>(L.P_total), bm)) return MOE_ERR_CUDA;
    a.out = pre;
    a.out_ld = n1;
    a.K = d;
    a.n_out = F;
    a.up_row_offset = F;
    a.acc = acc;
    a.acc_elems = static_cast<int64_t>(T) * d;
    a.zero2 = dtopk_weights;
    a.zero2_elems = dtopk_weights ? static_cast<int64_t>(T) * k : 0;
    StageScope scope(9, s);
    err = moe::launch_grouped_gemm(epi, a, grid_for(moe::gemm_max_tiles(epi, max_routed_blocks, n_shared_blocks, F)),
                                   s);
    if (err != cudaSuccess) return MOE_ERR_CUDA;
    ++launches;
  }
  // 3. dh = W2^T dout rows, and in its epilogue da (from the
  //    pre-activations), w * h and dL/d topk_weights
  {
    moe::GemmArgs a;
    base_args(a);
    const int epi = act == MOE_ACT_SWIGLU ? moe::kEpiGradSwiGLU : moe::kEpiGradRelu2;
    // W2 [E, d, F] read MN-major: {F (contiguous), d rows, E}, boxes of 64 x 64
    if (!encode_3d(&a.tm_w, w2, F, d, E, 64)) return MOE_ERR_CUDA;
    if (n_shared) {
      if (!encode_3d(&a.tm_ws, w2_shared, F, d, 1, 64)) return MOE_ERR_CUDA;
    } else {
      a.tm_ws = a.tm_w;
    }
    if (!encode_2d(&a.tm_x, gs, d, static_cast<uint64_t>(L.P_total), bm)) return MOE_ERR_CUDA;
    a.pre = pre;
    a.out = da;
    a.out_ld = n1;
    a.hw = hw;
    a.dtopk = dtopk_weights;
    a.K = d;
    a.n_out = F;
    a.up_row_offset = F;
    StageScope scope(10, s);
    err = moe::launch_grouped_gemm(epi, a, grid_for(moe::gemm_max_tiles(epi, max_routed_blocks, n_shared_blocks, F)),
                                   s);
    if (err != cudaSuccess) return MOE_ERR_CUDA;
    ++launches;
  }
  // 4. dx rows = W13^T da, added into the fp32 accumulator at their token;
  //    then dx = bf16(accumulator)
  {
    moe::GemmArgs a;
    base_args(a);
    // W13 [E, n1, d] read MN-major: {d (contiguous), n1 rows, E}, boxes of 64 x 64
    if (!encode_3d(&a.tm_w, w13, d, n1, E, 64)) return MOE_ERR_CUDA;
    if (n_shared) {
      if (!encode_3d(&a.tm_ws, w13_shared, d, n1, 1, 64)) return MOE_ERR_CUDA;
    } else {
      a.tm_ws = a.tm_w;
    }
    if (!encode_2d(&a.tm_x, da, n1, static_cast<uint64_t>(L.P_total), bm)) return MOE_ERR_CUDA;
    a.acc = acc;
    a.acc_elems = static_cast<int64_t>(T) * d;
    a.K = n1;
    a.n_out = d;
    {
      const int64_t acc_bytes = static_cast<int64_t>(T) * d * 4;
      const int64_t budget = int64_t(48) << 20;
      const int n_wt = (d + 255) / 256;
      const int passes = static_cast<int>((acc_bytes + budget - 1) / budget);
      a.pass_cols = passes <= 1 ? 0 : (n_wt + passes - 1) / passes;
    }
    StageScope scope(11, s);
    err = moe::launch_grouped_gemm(moe::kEpiDx, a,
                                   grid_for(moe::gemm_max_tiles(moe::kEpiDx, max_routed_blocks, n_shared_blocks, d)), s);
    if (err != cudaSuccess) return MOE_ERR_CUDA;
    ++launches;
  }
  {
    StageScope scope(4, s);
    err = moe::launch_convert(acc, static_cast<int64_t>(T) * d, dx, num_sms, s, &launches);
    if (err != cudaSuccess) return MOE_ERR_CUDA;
  }
  // 5. weight gradients per expert: dW13_e = da_e^T x_e, dW2_e = dout_e^T (w h)_e
  auto wgrad = [&](const uint16_t* A, int M, const uint16_t* B, int N, uint16_t* out, uint16_t* out_shared,
                   int stage) -> moe_status {
    moe::WgradArgs w;
    std::memset(&w, 0, sizeof(w));
    if (!encode_2d(&w.tm_a, A, M, static_cast<uint64_t>(L.P_total), 64)) return MOE_ERR_CUDA;
    if (!encode_2d(&w.tm_b, B, N, static_cast<uint64_t>(L.P_total), 64)) return MOE_ERR_CUDA;
    w.expert_ids = expert_ids;
    w.ntpp = num_tokens_post_padded;
    w.out = out;
    w.out_shared = out_shared;
    w.status = dev_status;
    w.wait_ns = wait_ns;
    w.E = E;
    w.M = M;
    w.N = N;
    w.block_m = bm;
    w.max_routed_blocks = max_routed_blocks;
    w.n_shared_blocks = n_shared_blocks;
    StageScope scope(stage, s);
    if (moe::launch_wgrad(w, grid_for(moe::wgrad_max_tiles(E, n_shared, M, N)), s) != cudaSuccess)
      return MOE_ERR_CUDA;
    ++launches;
    return MOE_OK;
  };
  st = wgrad(da, n1, xs, d, dw13, dw13_shared, 12);
  if (st != MOE_OK) return st;
  st = wgrad(gs, d, hw, F, dw2, dw2_shared, 13);
  if (st != MOE_OK) return st;
  return finish(cudaSuccess, launches);
}

moe_status moe_read_status(const int32_t* dev_status, moe_stream_t stream) {
  if (dev_status == nullptr) return MOE_ERR_INVALID_ARG;
  int32_t v = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&v, dev_status, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  return static_cast<moe_status>(v);
}

const char* moe_status_string(moe_status status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_NONFINITE: return "MOE_ERR_NONFINITE";
    case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT";
    case MOE_ERR_BAD_EXPERT_ID: return "MOE_ERR_BAD_EXPERT_ID";
  }
  return "MOE_ERR_UNKNOWN";
}

int moe_last_launch_count(void) { return g_last_launches; }

moe_status moe_debug_timeouts(uint64_t wait_limit_ns, int unreachable_arrivals) {
  if (unreachable_arrivals < 0 || unreachable_arrivals > 1024) return MOE_ERR_INVALID_ARG;
  moe::g_wait_limit_ns.store(wait_limit_ns == 0 ? moe::kWaitLimitNs : wait_limit_ns, std::memory_order_relaxed);
  moe::g_unreachable.store(unreachable_arrivals, std::memory_order_relaxed);
  return MOE_OK;
}

moe_status moe_profile_enable(int on) {
  if (on) release_records();  // a fresh record; disabling keeps the records readable
  g_profile = on != 0;
  while (g_profile && g_event_pool.size() < kEventPoolPrime) {
    cudaEvent_t ev;
    if (cudaEventCreate(&ev) != cudaSuccess) return MOE_ERR_CUDA;
    g_event_pool.push_back(ev);
  }
  return MOE_OK;
}

moe_status moe_profile_collect(double* stage_ms, int* stage_calls, int n_stages, int release) {
  if (stage_ms == nullptr || n_stages < 0) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < n_stages; ++i) {
    stage_ms[i] = 0.0;
    if (stage_calls) stage_calls[i] = 0;
  }
  moe_status st = MOE_OK;
  for (auto& r : g_records) {
    float ms = 0.0f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) {
      st = MOE_ERR_CUDA;
      continue;
    }
    if (r.stage >= 0 && r.stage < n_stages) {
      stage_ms[r.stage] += ms;
      if (stage_calls) ++stage_calls[r.stage];
    }
  }
  if (release) release_records();
  return st;
}

}  // extern "C"
