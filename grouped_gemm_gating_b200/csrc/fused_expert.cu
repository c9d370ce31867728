// Fused expert kernel for small token blocks (block_m = 16..64): gate/up GEMM
// with its activation, down GEMM with the top-k weights and the
// scatter-reduce, in one persistent launch.
//
// The computation is the layer of the fused-moe-kernel page ("Fused MoE
// Kernel Optimization": "Grouped GEMM Structure", "Common Pitfalls" 4) and of
// the axolotl `_moe_triton_forward` (src/axolotl/monkeypatch/deepseek_v3/
// __init__.py: gate/up projections, act_fn(gate) * up, down projection,
// weighted sum over the k experts), with the relu^2 experts of the mlxcel PR
// ("fc1 -> relu^2 -> fc2").  For the decode / verifier shape the layer is
// bound by streaming each hit expert's weights once, so the design avoids
// anything that stalls that stream.
//
// Split along d_ff.  A tile is (block of block_m token rows, one slice of
// 128 h columns).  A CTA
//   1. computes the slice's pre-activations with the weights as the MMA's
//      M = 128 rows (SwiGLU: the 128 gate rows and the matching 128 up rows
//      of each K block are two stages, multiplied into two accumulators),
//   2. writes h = act(...) for the slice into shared memory, already in the
//      K-major 128-byte-swizzled layout the tensor core reads,
//   3. streams the matching columns of W2 (256 contiguous bytes of every
//      row, as two 64-column K blocks) for every 128-row d tile and
//      multiplies them by that h slice,
//   4. adds topk_weight * partial into an fp32 [T, d] accumulator with
//      red.global.add (fire-and-forget).
// No tile waits for another CTA's work while weights stream (a GPU-scope
// handoff from an SM whose TMA queue is full takes several microseconds).
// The fp32 partials are summed in an order that depends on timing, so the
// output is reproducible to fp32 rounding of the sum, not bit for bit.
//
// Each CTA runs its tiles software-pipelined: gate/up of tile i+1 is issued
// before the down GEMM of tile i, so the tensor core never idles while the
// epilogue turns tile i's accumulator into its h slice.
//
// Grid protocol (all CTAs co-resident: one per SM, grid <= SM count):
//   start: the gather warps zero this CTA's slice of the accumulator and
//          count the CTA on sync[0]; the epilogue waits for all CTAs there
//          before its first reduction (the weight stream does not wait).
//   end:   every CTA counts itself on sync[1] once its reductions are issued;
//          the last to arrive zeroes sync[0..1].  For a small output (T*d <=
//          16384) that CTA converts the whole accumulator to bf16 and the
//          others have already left.  Otherwise it moves the generation in
//          sync[2] on by one, which releases the others (each read it before
//          counting itself), and every CTA converts its slice of the
//          accumulator.  A CTA that gave up on a wait counts itself and
//          leaves, so sync[0..1] are zero after every launch, timeouts
//          included, and sync[2] only ever moves forward.
//
// Tiles are dealt to the fewest CTAs that can take equal shares; the other
// CTAs only zero and convert their slice of the accumulator.
//
// Warp roles: warp 0 TMA producer (weights), warp 1 TMEM allocator + MMA
// issuer, warps 2-5 epilogue, warps 6-9 token-row gather (cp.async; each
// thread's copies arrive on the stage's full barrier when they land).  TMEM:
// the gate/up accumulators of two tiles in flight (block_m columns each;
// SwiGLU has a gate and an up accumulator per tile), then a ring of
// down-GEMM accumulators (groups of 64 columns).  Every wait is bounded in
// time; on expiry the kernel records MOE_ERR_DEVICE_TIMEOUT and all roles
// leave.
#include <cuda_fp16.h>

#include <atomic>

#include "align_impl.cuh"
#include "common.cuh"
#include "fused.h"
#include "gemm.h"
#include "ptx.cuh"
#include "route_impl.cuh"

namespace moe {

namespace {

// In-kernel routing limit (block_m = 16 only): T*k <= 256 slots.
constexpr int kRouteMaxS = 256;
// Outputs of at most this many elements (T * d) are converted to bf16 by the
// last CTA to finish, alone: the others leave without waiting for a release.
constexpr int kLastCtaConvertMax = 16384;

template <int EPI1, int TOK, bool ROUTE, bool FP8 = false>
struct FusedCfg {
  static constexpr bool kGated = (EPI1 == kEpiSwiGLU);
  static constexpr int kH = 128;                // h columns per tile
  static constexpr int kHk = kH / 64;           // 64-wide K blocks of the down GEMM per tile
  // gate/up stages per 64-wide K block: SwiGLU loads the slice's 128 gate
  // rows and then its 128 up rows, each multiplied into its own accumulator
  static constexpr int kGU = kGated ? 2 : 1;
  static constexpr int kAcc1 = kGU * TOK;       // TMEM columns of one tile's gate/up accumulator(s)
  static constexpr int kBoxRows = kGated ? kFusedBoxRowsGated : kFusedBoxRowsRelu2;
  static constexpr int kWBytes = 128 * 128;     // 128 weight rows x 64 bf16 per stage
  static constexpr int kXBytes = TOK * 128;     // token rows x 64 bf16 per stage
  static constexpr int kStageBytes = kWBytes + kXBytes;
  static constexpr int kHBufBytes = kHk * TOK * 128;            // one h slice (B operand of the down GEMM)
  static constexpr int kTokBytes = 2 * 2 * 64 * 4;              // token id and weight per row, two tiles
  static constexpr int kBarrierBytes = 1024;
  // routing results kept for the whole kernel: expert and weight of every
  // slot, its rank among its expert's slots, the slots in expert order, and
  // per expert its slot count and padded / unpadded offsets
  static constexpr int kRouteBytes = ROUTE ? (4 * kRouteMaxS + 3 * (MOE_MAX_EXPERTS + 1) + 5) * 4 : 0;
  static constexpr int kFixedBytes = 2 * kHBufBytes + kTokBytes + kBarrierBytes + kRouteBytes + 1024;
  static constexpr int kStagesRaw = (227 * 1024 - kFixedBytes) / kStageBytes;
  // fp8 weights: the weight stream lands in a deeper ring of raw stages (128
  // rows x 64 e4m3 bytes and the 2 x 128 scale bytes of those rows), which
  // the converter warps expand into a short ring of bf16 operand stages
  static constexpr int kStages = FP8 ? 4 : (kStagesRaw > 12 ? 12 : kStagesRaw);
  static constexpr int kRawWBytes = 128 * 64;
  static constexpr int kRawStageBytes = kRawWBytes + 256;
  static constexpr int kRawRoom = 227 * 1024 - kFixedBytes - kStages * kStageBytes - 1024;
  static constexpr int kRawStages = FP8 ? (kRawRoom / kRawStageBytes > 16 ? 16 : kRawRoom / kRawStageBytes) : 0;
  static constexpr int kRawRegion = (kRawStages * kRawStageBytes + 1023) / 1024 * 1024;
  // Down-GEMM accumulators: groups of kGroup d tiles (64 TMEM columns) form
  // one slot of a TMEM ring, so the epilogue synchronises once per group.
  static constexpr int kGroup = 64 / TOK;
  static constexpr int kD2Raw = (512 - 2 * kAcc1) / 64;
  static constexpr int kD2Slots = kD2Raw > 8 ? 8 : kD2Raw;
  // warps: producer, MMA, 4 epilogue, 4 gather (+ 4 converters for fp8 weights)
  static constexpr int kNumThreads = FP8 ? 448 : 320;
  static constexpr int kSmemBytes = kStages * kStageBytes + kRawRegion + kFixedBytes;
  static constexpr uint32_t kIdesc = ptx::idesc_bf16_f32(128, TOK);
  static_assert(TOK == 16 || TOK == 32 || TOK == 64, "token rows per tile");
  static_assert(kStageBytes % 1024 == 0 && kHBufBytes % 1024 == 0, "1024-byte aligned operand tiles");
  static_assert(kStages >= 3, "pipeline depth");
  // every box starts on a 1024-byte swizzle atom (8 rows of 128 B) of the operand
  static_assert(128 % kFusedBoxRowsGated == 0 && 128 % kFusedBoxRowsRelu2 == 0 && 128 % kFusedBoxRowsW2 == 0 &&
                    kFusedBoxRowsGated % 8 == 0 && kFusedBoxRowsRelu2 % 8 == 0 && kFusedBoxRowsW2 % 8 == 0,
                "weight boxes tile the 128-row operand on swizzle-atom boundaries");
  static_assert((2 * kStages + 9 + 2 * kD2Slots + 2 * kRawStages) * 8 + 16 <= kBarrierBytes, "barrier area");
  static_assert(!FP8 || kRawStages >= 6, "fp8 raw-stage ring depth");
  static_assert(kSmemBytes <= 232448, "shared memory per block");
};

struct TileInfo {
  int blk, wt;
  bool shared_blk;
};

__device__ __forceinline__ TileInfo tile_info(int u, int n_h, int routed_blocks) {
  TileInfo t;
  t.blk = u / n_h;
  t.wt = u - t.blk * n_h;
  t.shared_blk = t.blk >= routed_blocks;
  return t;
}

// silu(g) = g * sigmoid(g); the quotient with the fast approximate divide
// (h is rounded to bf16 right after, far coarser than its error).
__device__ __forceinline__ float silu_fast(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// The d tiles of a tile's down GEMM are walked starting at a tile-dependent
// offset, so that CTAs working at the same time add into different lines of
// the accumulator instead of all hitting the same ones.
__device__ __forceinline__ int d_rotation(int u, int n_d) { return u % n_d; }
__device__ __forceinline__ int d_tile(int k, int rot, int n_d) {
  const int di = k + rot;
  return di >= n_d ? di - n_d : di;
}

__device__ __forceinline__ void red_add_f32(float* p, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Two e4m3 values (the low 16 bits of `two`, element 0 in the low byte)
// times `scale`, as two bf16 (element 0 in the low half).  e4m3 -> f16 is
// exact, and so is the product with a power of two within range.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t two, float scale) {
  uint32_t h;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(h) : "r"(two));
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
  return pack_bf16x2(f.x * scale, f.y * scale);
}

// Named barrier 1 over the four epilogue warps, 2 over the four gather warps
// (barrier 0 is __syncthreads).  Each warp reconverges first, as the aligned
// barrier requires.  epilogue_any() is barrier 1 with an OR reduction: the
// epilogue takes every leave-on-timeout decision uniformly, so no epilogue
// thread can be left waiting at a later barrier for one that left.
__device__ __forceinline__ void epilogue_sync() {
  __syncwarp();
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

__device__ __forceinline__ void gather_sync() {
  __syncwarp();
  asm volatile("bar.sync 2, 128;" ::: "memory");
}

// Named barrier 4 over the producer warp and the four gather warps, at exit.
__device__ __forceinline__ void exit_handshake() {
  __syncwarp();
  asm volatile("bar.sync 4, 160;" ::: "memory");
}

__device__ __forceinline__ bool epilogue_any(bool v) {
  uint32_t r;
  __syncwarp();
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(v ? 1u : 0u)
      : "memory");
  return r != 0;
}

// Bounded spin until *p != v (acquire).  False on timeout.
__device__ __forceinline__ bool spin_until_changed(const int32_t* p, int v, uint64_t limit_ns) {
  const uint64_t t0 = ptx::globaltimer_ns();
  while (ptx::ld_acquire_gpu(p) == v) {
    if (ptx::globaltimer_ns() - t0 > limit_ns) return false;
    __nanosleep(64);
  }
  return true;
}

// Bounded spin until *p >= target (acquire).  False on timeout or abort.
__device__ __forceinline__ bool spin_until(const int32_t* p, int target, volatile int* abort_flag,
                                           uint64_t limit_ns) {
  const uint64_t t0 = ptx::globaltimer_ns();
  while (ptx::ld_acquire_gpu(p) < target) {
    if (*abort_flag || ptx::globaltimer_ns() - t0 > limit_ns) return false;
    __nanosleep(64);
  }
  return true;
}

template <int EPI1, int TOK, bool ROUTE, bool FP8>
__global__ void __launch_bounds__(FusedCfg<EPI1, TOK, ROUTE, FP8>::kNumThreads, 1)
    fused_expert_kernel(const __grid_constant__ FusedArgs args) {
  using C = FusedCfg<EPI1, TOK, ROUTE, FP8>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* raw = smem + C::kStages * C::kStageBytes;         // fp8 only: [kRawStages][weights | scales]
  uint8_t* hbuf = raw + C::kRawRegion;                        // [2][kHk][TOK rows x 128 B]
  int* tok_s = reinterpret_cast<int*>(hbuf + 2 * C::kHBufBytes);  // [2][64]
  float* w_s = reinterpret_cast<float*>(tok_s + 2 * 64);                           // [2][64]
  uint64_t* full = reinterpret_cast<uint64_t*>(w_s + 2 * 64);
  uint64_t* empty = full + C::kStages;
  uint64_t* d1_full = empty + C::kStages;
  uint64_t* d1_empty = d1_full + 2;
  uint64_t* hb_full = d1_empty + 2;
  uint64_t* hb_empty = hb_full + 2;
  uint64_t* mma_done = hb_empty + 2;
  uint64_t* d2_full = mma_done + 1;
  uint64_t* d2_empty = d2_full + C::kD2Slots;
  uint64_t* raw_full = d2_empty + C::kD2Slots;    // fp8: the raw stage's bytes landed
  uint64_t* raw_empty = raw_full + C::kRawStages;  // fp8: the converters are done with it
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(raw_empty + C::kRawStages);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* flag = reinterpret_cast<volatile int*>(tmem_holder + 2);
  volatile int* prod_issued = reinterpret_cast<volatile int*>(tmem_holder + 3);  // stages the producer filled

  const int warp = threadIdx.x / kWarp;
  const int lane = threadIdx.x % kWarp;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      // bf16 weights: the producer's bytes and the gather warps' rows; fp8:
      // the converter threads' expanded weights and the gather warps' rows
      ptx::mbar_init(&full[s], FP8 ? 128 + 128 : 1 + 128);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < C::kRawStages; ++s) {
      ptx::mbar_init(&raw_full[s], 1);
      ptx::mbar_init(&raw_empty[s], 4);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&d1_full[b], 1);
      ptx::mbar_init(&d1_empty[b], 4);
      ptx::mbar_init(&hb_full[b], 1);
      ptx::mbar_init(&hb_empty[b], 1);
    }
    ptx::mbar_init(mma_done, 1);
    for (int s = 0; s < C::kD2Slots; ++s) {
      ptx::mbar_init(&d2_full[s], 1);
      ptx::mbar_init(&d2_empty[s], 4);
    }
    *abort_flag = 0;
    *flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&args.tm_w13);
    ptx::prefetch_tmap(&args.tm_w2);
    if (args.n_shared_blocks) {
      ptx::prefetch_tmap(&args.tm_w13s);
      ptx::prefetch_tmap(&args.tm_w2s);
    }
    if (FP8) {
      ptx::prefetch_tmap(&args.tm_s13);
      ptx::prefetch_tmap(&args.tm_s2);
    }
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_holder, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  pdl_wait();
  pdl_launch_dependents();
  // routing results in shared memory (in-kernel routing only)
  int* r_ids = nullptr;      // [S] expert of each slot
  float* r_w = nullptr;      // [S] its weight
  int* r_rank = nullptr;     // [S] rank of the slot among its expert's slots
  int* r_compact = nullptr;  // [S] slots in (expert, slot) order
  int* r_cnt = nullptr;      // [E] slots per expert
  int* r_off = nullptr;      // [E + 1] padded offsets (r_off[E] = padded total)
  int* r_coff = nullptr;     // [E + 1] unpadded offsets
  int ntpp_v;
  if constexpr (ROUTE) {
    // ---- routing of all tokens and their per-expert order, redundantly in
    // every CTA, before any weight streams: counts, two scans and a rank per
    // slot are all the kernel needs (a block's expert and a row's slot are
    // looked up from them); the padded sort itself is only written out, by
    // CTA 0's epilogue warps while the first weights stream.
    r_ids = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(full) + C::kBarrierBytes);
    r_w = reinterpret_cast<float*>(r_ids + kRouteMaxS);
    r_rank = reinterpret_cast<int*>(r_w + kRouteMaxS);
    r_compact = r_rank + kRouteMaxS;
    r_cnt = r_compact + kRouteMaxS;
    r_off = r_cnt + MOE_MAX_EXPERTS + 1;
    r_coff = r_off + MOE_MAX_EXPERTS + 1;
    constexpr int kWarps = C::kNumThreads / kWarp;
    float* gscore = reinterpret_cast<float*>(smem);  // [kWarps][64] on the idle stage ring
    unsigned char* gkeep = reinterpret_cast<unsigned char*>(gscore + kWarps * 64);  // [kWarps][64]
    const FusedRoute& R = args.route;
    for (int i = threadIdx.x; i < args.E; i += C::kNumThreads) r_cnt[i] = 0;
    for (int t = warp; t < args.T; t += kWarps) {
      const float* row = R.logits + static_cast<size_t>(t) * args.E;
      if (args.E <= 128)
        route_one_token<4>(row, args.E, args.k, R.n_group, R.topk_group, R.group_score, R.renormalize,
                           R.routed_scaling, gscore + warp * 64, gkeep + warp * 64, r_ids + t * args.k,
                           r_w + t * args.k, args.status, lane);
      else
        route_one_token<8>(row, args.E, args.k, R.n_group, R.topk_group, R.group_score, R.renormalize,
                           R.routed_scaling, gscore + warp * 64, gkeep + warp * 64, r_ids + t * args.k,
                           r_w + t * args.k, args.status, lane);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < args.S; i += C::kNumThreads) atomicAdd(&r_cnt[r_ids[i]], 1);
    __syncthreads();
    if (warp == 0) align_detail::warp_padded_scan(r_cnt, r_off, args.E, args.block_m, lane);
    if (warp == 1) align_detail::warp_padded_scan(r_cnt, r_coff, args.E, 1, lane);
    __syncthreads();  // the stage ring is free again
    // The weight producer and the MMA issuer need only the counts and the
    // padded offsets: they start streaming now, while the epilogue and
    // gather warps rank the slots (for row -> slot lookups) and meet at
    // named barrier 3.
    if (warp >= 2) {
      for (int i = static_cast<int>(threadIdx.x) - 64; i < args.S; i += C::kNumThreads - 64) {
        const int e = r_ids[i];
        int rank = 0;
        for (int j = 0; j < i; ++j) rank += r_ids[j] == e ? 1 : 0;
        r_rank[i] = rank;
        r_compact[r_coff[e] + rank] = i;
      }
      __syncwarp();
      asm volatile("bar.sync 3, %0;" ::"r"(C::kNumThreads - 64) : "memory");
    }
    ntpp_v = r_off[args.E];
  } else {
    ntpp_v = *args.ntpp;
  }
  // expert of routed block `blk`, and the slot of row j of it (S: padding)
  auto block_exp = [&](int blk) -> int {
    if constexpr (ROUTE) {
      return align_detail::block_expert(r_off, args.E, blk * args.block_m);
    } else {
      return args.expert_ids[blk];
    }
  };
  auto row_slot = [&](int blk, int e, int j) -> int {
    if constexpr (ROUTE) {
      const int i = blk * args.block_m + j - r_off[e];
      return i < r_cnt[e] ? r_compact[r_coff[e] + i] : args.S;
    } else {
      return args.sorted_ids[blk * args.block_m + j];
    }
  };
  auto slot_weight = [&](int slot) -> float {
    if constexpr (ROUTE) {
      return r_w[slot];
    } else {
      return args.topk_w[slot];
    }
  };
  int routed_blocks = ntpp_v / args.block_m;
  if (routed_blocks < 0) routed_blocks = 0;
  if (routed_blocks > args.max_routed_blocks) routed_blocks = args.max_routed_blocks;
  const int total_blocks = routed_blocks + args.n_shared_blocks;
  const int n_h = (args.F + C::kH - 1) / C::kH;
  const int n_d = (args.d + 127) / 128;
  const int total_tiles = total_blocks * n_h;
  // Tiles are dealt to the fewest CTAs that can each take the per-CTA
  // maximum: with 252 tiles on 148 CTAs, 126 CTAs take two tiles each
  // instead of 104 taking two and 44 taking one.  Every CTA streams the same
  // bytes and gets a larger share of HBM while it streams.  The other CTAs
  // only zero and convert their share of the accumulator.
  // Tiles of this CTA: blockIdx.x, blockIdx.x + tile_stride, ...
  const int tiles_per_cta = (total_tiles + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x);
  const int tile_stride = tiles_per_cta > 0 ? (total_tiles + tiles_per_cta - 1) / tiles_per_cta : 1;
  const int n_my = static_cast<int>(blockIdx.x) < tile_stride
                       ? (total_tiles - static_cast<int>(blockIdx.x) + tile_stride - 1) / tile_stride
                       : 0;
  const int nk1 = args.d / 64;
  const int nk2 = n_d * C::kHk;  // down-GEMM stages per tile
  const int ng = nk1 * C::kGU;   // gate/up stages per tile
  const int nacc = args.T * args.d;

  auto fail = [&]() {
    *abort_flag = 1;
    set_status(args.status, MOE_ERR_DEVICE_TIMEOUT);
  };
  auto tile_of = [&](int i) { return tile_info(static_cast<int>(blockIdx.x) + i * tile_stride, n_h, routed_blocks); };

  // Stage order of every role: gate/up of tile 0; then for i >= 1 gate/up of
  // tile i followed by the down GEMM of tile i-1; last the down GEMM of the
  // final tile.
  if (warp == 0) {
    // ------------------------------------------------ TMA producer (weights)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      auto expert_of = [&](const TileInfo& t) {
        if (t.shared_blk) return 0;
        const int e = block_exp(t.blk);
        if (e < 0 || e >= args.E) set_status(args.status, MOE_ERR_BAD_EXPERT_ID);  // TMA fills zeros
        return e;
      };
      // the ring this producer fills: the bf16 operand stages, or for fp8
      // weights the raw stages (whose slots the converters hand back)
      constexpr int kRing = FP8 ? C::kRawStages : C::kStages;
      uint64_t* ring_free = FP8 ? raw_empty : empty;
      auto acquire = [&]() {
        if (!ptx::mbar_wait_bounded(&ring_free[stage], phase ^ 1u, abort_flag, args.wait_ns)) {
          fail();
          ok = false;
        }
        return ok;
      };
      int issued = 0;  // stages filled so far
      auto advance = [&]() {
        ++issued;
        if (++stage == kRing) {
          stage = 0;
          phase ^= 1u;
        }
      };
      // fp8: one stage = 128 weight rows x 64 e4m3 bytes and the scale bytes
      // of those rows for the stage's two 32-wide K blocks
      auto load_raw = [&](const CUtensorMap* tw, const CUtensorMap* ts, int kcol, int row0, int e, uint64_t pol) {
        uint8_t* rb = raw + stage * C::kRawStageBytes;
        ptx::mbar_arrive_expect_tx(&raw_full[stage], C::kRawStageBytes);
        ptx::tma_load_3d_hint(rb, tw, &raw_full[stage], kcol, row0, e, pol);
        ptx::tma_load_3d_hint(rb + C::kRawWBytes, ts, &raw_full[stage], row0, kcol / 32, e, pol);
      };
      // Streamed weight lines are used once: mark them first to leave L2.
      const uint64_t evict_first = ptx::l2_policy_evict_first();
      for (int i = 0; ok && i <= n_my; ++i) {
        if (i < n_my) {
          const TileInfo t = tile_of(i);
          const int e = expert_of(t);
          const CUtensorMap* tm = t.shared_blk ? &args.tm_w13s : &args.tm_w13;
          for (int s = 0; s < ng && acquire(); ++s) {
            // K block s / kGU; SwiGLU: gate rows [wt*128, +128), then up rows [F + wt*128, +128)
            const int kb = s / C::kGU;
            const int row0 = (C::kGated && s != kb * C::kGU ? args.F : 0) + t.wt * C::kH;
            if constexpr (FP8) {
              load_raw(tm, t.shared_blk ? &args.tm_s13s : &args.tm_s13, kb * 64, row0, e, evict_first);
            } else {
              uint8_t* sW = smem + stage * C::kStageBytes;
              ptx::mbar_arrive_expect_tx(&full[stage], C::kWBytes);
#pragma unroll
              for (int r = 0; r < 128; r += C::kBoxRows)
                ptx::tma_load_3d_hint(sW + r * 128, tm, &full[stage], kb * 64, row0 + r, e, evict_first);
            }
            advance();
          }
        }
        if (ok && i >= 1) {
          const TileInfo t = tile_of(i - 1);
          const int e = expert_of(t);
          const CUtensorMap* tm = t.shared_blk ? &args.tm_w2s : &args.tm_w2;
          const int rot = d_rotation(static_cast<int>(blockIdx.x) + (i - 1) * tile_stride, n_d);
          for (int s = 0; s < nk2 && acquire(); ++s) {
            const int dk = s / C::kHk, kk = s - dk * C::kHk;
            const int di = d_tile(dk, rot, n_d);
            if constexpr (FP8) {
              load_raw(tm, t.shared_blk ? &args.tm_s2s : &args.tm_s2, t.wt * C::kH + kk * 64, di * 128, e,
                       evict_first);
            } else {
              uint8_t* sW = smem + stage * C::kStageBytes;
              ptx::mbar_arrive_expect_tx(&full[stage], C::kWBytes);
#pragma unroll
              for (int r = 0; r < 128; r += kFusedBoxRowsW2)
                ptx::tma_load_3d_hint(sW + r * 128, tm, &full[stage], t.wt * C::kH + kk * 64, di * 128 + r, e,
                                      evict_first);
            }
            advance();
          }
        }
      }
      *prod_issued = issued;
    }
    // The last load into every stage lands before the CTA's shared memory is
    // released.  After an abort some were never consumed.  bf16 weights: a
    // stage's phase completes only with the gather warps' arrivals too, so
    // they add the ones they did not make (exit_handshake); fp8 weights: the
    // raw stages complete on the loaded bytes alone.  Then the producer
    // waits for the last phase of every stage it filled (at once after a
    // normal run, where they have all been consumed).
    if constexpr (!FP8) {
      exit_handshake();
      exit_handshake();
    }
    if (lane == 0) {
      constexpr int kRing = FP8 ? C::kRawStages : C::kStages;
      uint64_t* ring_full = FP8 ? raw_full : full;
      const int issued = *prod_issued;
      int stage = issued % kRing;
      uint32_t phase = static_cast<uint32_t>((issued / kRing) & 1);
      for (int j = 1; j <= kRing && j <= issued; ++j) {
        int st = stage - j;
        uint32_t ph = phase;
        if (st < 0) {
          st += kRing;
          ph ^= 1u;
        }
        ptx::mbar_wait_bounded(&ring_full[st], ph, flag, kDrainLimitNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int d2c = 0;
      bool ok = true;
      auto wait = [&](uint64_t* bar, uint32_t parity) {
        if (!ptx::mbar_wait_bounded(bar, parity, abort_flag, args.wait_ns)) {
          fail();
          ok = false;
        }
        return ok;
      };
      for (int i = 0; ok && i <= n_my; ++i) {
        if (i < n_my) {
          const int b = i & 1;
          const uint32_t bph = static_cast<uint32_t>((i >> 1) & 1);
          if (!wait(&d1_empty[b], bph ^ 1u)) break;
          ptx::tc_fence_after();
          const uint32_t d1 = tmem_base + static_cast<uint32_t>(b * C::kAcc1);
          for (int s = 0; s < ng; ++s) {
            if (!wait(&full[stage], phase)) break;
            ptx::tc_fence_after();
            ptx::fence_proxy_async_smem();  // token rows were written by cp.async
            const int kb = s / C::kGU;
            const uint32_t acc = d1 + static_cast<uint32_t>((s - kb * C::kGU) * TOK);  // gate or up accumulator
            const uint32_t sW = ptx::smem_u32(smem + stage * C::kStageBytes);
            const uint32_t sX = sW + C::kWBytes;
#pragma unroll
            for (int q = 0; q < 4; ++q)
              ptx::mma_bf16(acc, ptx::sw128_kmajor_desc(sW + q * 32), ptx::sw128_kmajor_desc(sX + q * 32), C::kIdesc,
                            (kb | q) != 0 ? 1u : 0u);
            ptx::mma_commit(&empty[stage]);
            if (++stage == C::kStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          ptx::mma_commit(&d1_full[b]);
        }
        if (i >= 1) {
          const int p = i - 1;
          const int b = p & 1;
          if (!wait(&hb_full[b], static_cast<uint32_t>((p >> 1) & 1))) break;
          ptx::tc_fence_after();
          const uint32_t sH = ptx::smem_u32(hbuf + b * C::kHBufBytes);
          const int n_g = (n_d + C::kGroup - 1) / C::kGroup;
          for (int g = 0; ok && g < n_g; ++g, ++d2c) {
            const int slot = d2c % C::kD2Slots;
            const uint32_t sph = static_cast<uint32_t>((d2c / C::kD2Slots) & 1);
            if (!wait(&d2_empty[slot], sph ^ 1u)) break;
            ptx::tc_fence_after();
            for (int w = 0; ok && w < C::kGroup && g * C::kGroup + w < n_d; ++w) {
              const uint32_t d2 = tmem_base + static_cast<uint32_t>(2 * C::kAcc1 + slot * 64 + w * TOK);
              for (int kk = 0; kk < C::kHk; ++kk) {
                if (!wait(&full[stage], phase)) break;
                ptx::tc_fence_after();
                const uint32_t sW = ptx::smem_u32(smem + stage * C::kStageBytes);
                const uint32_t sB = sH + kk * TOK * 128;
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  ptx::mma_bf16(d2, ptx::sw128_kmajor_desc(sW + q * 32), ptx::sw128_kmajor_desc(sB + q * 32),
                                C::kIdesc, (kk | q) != 0 ? 1u : 0u);
                ptx::mma_commit(&empty[stage]);
                if (++stage == C::kStages) {
                  stage = 0;
                  phase ^= 1u;
                }
              }
            }
            if (!ok) break;
            ptx::mma_commit(&d2_full[slot]);
          }
          if (!ok) break;
          ptx::mma_commit(&hb_empty[b]);  // the h slice may be overwritten once these MMAs finish
        }
      }
      // no MMA of this CTA may still run when TMEM is freed (this wait
      // ignores the abort flag; *flag stays zero until the block barrier)
      ptx::mma_commit(mma_done);
      if (!ptx::mbar_wait_bounded(mma_done, 0u, flag, kDrainLimitNs)) fail();
    }
  } else if (warp < 6) {
    // ------------------------------------------------ epilogue
    const int q = warp & 3;         // TMEM lane quadrant this warp may access
    const int row = q * 32 + lane;  // accumulator row: weight row / d row within the tile
    const int etid = threadIdx.x - 64;
    if constexpr (ROUTE) {
      if (blockIdx.x == 0) {  // the outputs of the separate routing and align calls
        const FusedRoute& R = args.route;
        for (int i = etid; i < args.S; i += 128) {
          R.topk_ids[i] = r_ids[i];
          R.topk_w[i] = r_w[i];
          R.inv_pos[i] = r_off[r_ids[i]] + r_rank[i];
        }
        for (int p = etid; p < R.P_max; p += 128) {
          int v = args.S;
          if (p < ntpp_v) {
            const int e = align_detail::block_expert(r_off, args.E, p);
            const int i = p - r_off[e];
            if (i < r_cnt[e]) v = r_compact[r_coff[e] + i];
          }
          R.sorted_ids[p] = v;
        }
        for (int b = etid; b < R.P_max / args.block_m; b += 128)
          R.expert_ids[b] = align_detail::block_expert(r_off, args.E, b * args.block_m);
        if (etid == 0) *R.ntpp = ntpp_v;
      }
    }
    bool zero_seen = false;
    int d2c = 0;
    // Same order as the MMA: the gate/up accumulator of tile i is turned
    // into h before the down-GEMM partials of tile i-1 are reduced, so the
    // tensor core finds h(i) ready when it reaches the down GEMM of tile i.
    for (int i = 0; i <= n_my; ++i) {
      if (i < n_my) {
        const TileInfo t = tile_of(i);
        const int b = i & 1;
        const uint32_t bph = static_cast<uint32_t>((i >> 1) & 1);
        // token and weight of each row of the block (-1: padding), used by
        // the reduction of this tile one step later
        if (etid < TOK) {
          const int j = etid;
          int tok = -1;
          float wj = 0.0f;
          if (!t.shared_blk) {
            const int slot = row_slot(t.blk, block_exp(t.blk), j);
            if (static_cast<unsigned>(slot) < static_cast<unsigned>(args.S)) {
              tok = slot / args.k;
              wj = slot_weight(slot);
            }
          } else {
            const int tk = (t.blk - routed_blocks) * args.block_m + j;
            if (tk < args.T) {
              tok = tk;
              wj = 1.0f;
            }
          }
          tok_s[b * 64 + j] = tok;
          w_s[b * 64 + j] = wj;
        }
        const bool got = ptx::mbar_wait_bounded(&d1_full[b], bph, abort_flag, args.wait_ns) &&
                         ptx::mbar_wait_bounded(&hb_empty[b], bph ^ 1u, abort_flag, args.wait_ns);
        if (epilogue_any(!got)) {
          if (!got) fail();
          break;
        }
        ptx::tc_fence_after();
        // ---- gate/up accumulator(s) -> h slice in shared memory (MMA operand
        // layout).  Thread `row` owns h column row of the slice: the gate (or
        // fc1) row `row` and, for SwiGLU, the matching up row are its TMEM lane
        // in the two accumulators.
        const uint32_t t1 =
            tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(b * C::kAcc1);
        uint8_t* hb = hbuf + b * C::kHBufBytes;
        {
          const int c = row & 63, kk = row >> 6;  // h column within its 64-wide K block
          // a slice past d_ff (the last slice when F % 128 == 64) reads other
          // rows or zeros there: its h columns are set to zero
          const bool live = t.wt * C::kH + row < args.F;
#pragma unroll
          for (int j0 = 0; j0 < TOK; j0 += 16) {
            uint32_t a[16], u[16];
            ptx::tmem_ld16(t1 + j0, a);
            if (C::kGated) ptx::tmem_ld16(t1 + TOK + j0, u);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              asm volatile("" : "+r"(a[jj]));  // uses stay after the wait
              if (C::kGated) asm volatile("" : "+r"(u[jj]));
            }
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              const int j = j0 + jj;
              float v;
              if (C::kGated) {
                v = silu_fast(__uint_as_float(a[jj])) * __uint_as_float(u[jj]);
              } else {
                v = fmaxf(__uint_as_float(a[jj]), 0.0f);
                v *= v;
              }
              if (!live) v = 0.0f;
              const uint32_t off =
                  kk * TOK * 128 + (j >> 3) * 1024 + (j & 7) * 128 + (((c >> 3) ^ (j & 7)) << 4) + (c & 7) * 2;
              *reinterpret_cast<uint16_t*>(hb + off) = float_to_bf16_bits(v);
            }
          }
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&d1_empty[b]);
        }
        ptx::fence_proxy_async_smem();  // the tensor core reads the h slice next
        epilogue_sync();                // (also publishes tok_s / w_s of this tile)
        if (etid == 0) ptx::mbar_arrive(&hb_full[b]);
      }
      if (i >= 1) {
        const int p = i - 1;
        const int b = p & 1;
        // every CTA has zeroed its slice of the accumulator before anyone adds
        if (!zero_seen) {
          const bool got = etid != 0 || spin_until(args.sync, static_cast<int>(gridDim.x) + args.start_surplus,
                                                   abort_flag, args.wait_ns);
          if (epilogue_any(!got)) {
            if (!got) fail();
            break;
          }
          zero_seen = true;
        }
        // ---- down-GEMM partial of every d tile -> fp32 accumulator
        const int rot = d_rotation(static_cast<int>(blockIdx.x) + p * tile_stride, n_d);
        const int* tk = tok_s + b * 64;
        const float* wk = w_s + b * 64;
        // valid rows of a block come first (an expert's padding ends its
        // last block; shared-expert blocks end at row T), so the reduction
        // stops at the first padding row
        int n_valid = TOK;
#pragma unroll
        for (int j = TOK - 1; j >= 0; --j)
          if (tk[j] < 0) n_valid = j;
        bool left = false;
        const int n_g = (n_d + C::kGroup - 1) / C::kGroup;
        for (int g = 0; g < n_g; ++g, ++d2c) {
          const int slot = d2c % C::kD2Slots;
          const uint32_t sph = static_cast<uint32_t>((d2c / C::kD2Slots) & 1);
          const bool got = ptx::mbar_wait_bounded(&d2_full[slot], sph, abort_flag, args.wait_ns);
          if (epilogue_any(!got)) {
            if (!got) fail();
            left = true;
            break;
          }
          ptx::tc_fence_after();
          const int n_w = min(C::kGroup, n_d - g * C::kGroup);
          const uint32_t t2 =
              tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(2 * C::kAcc1 + slot * 64);
          uint32_t a[C::kGroup][TOK];
#pragma unroll
          for (int w = 0; w < C::kGroup; ++w) {
            if (w < n_w) {
#pragma unroll
              for (int j0 = 0; j0 < TOK; j0 += 16)
                ptx::tmem_ld16(t2 + w * TOK + j0, *reinterpret_cast<uint32_t(*)[16]>(&a[w][j0]));
            }
          }
          ptx::tmem_wait_ld();
#pragma unroll
          for (int w = 0; w < C::kGroup; ++w)
#pragma unroll
            for (int j = 0; j < TOK; ++j) asm volatile("" : "+r"(a[w][j]));  // uses stay after the wait
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&d2_empty[slot]);
#pragma unroll
          for (int w = 0; w < C::kGroup; ++w) {
            const int drow = d_tile(g * C::kGroup + w, rot, n_d) * 128 + row;
            if (w < n_w && drow < args.d) {
              float* dst = args.acc + drow;
#pragma unroll
              for (int j = 0; j < TOK; ++j) {
                if (j >= n_valid) break;
                red_add_f32(dst + static_cast<size_t>(tk[j]) * args.d, wk[j] * __uint_as_float(a[w][j]));
              }
            }
          }
        }
        if (left) break;
        epilogue_sync();  // all reads of this tok_s / w_s buffer are done before it is rewritten
      }
    }
  } else if (warp < 10) {
    // ------------------------------------------------ token-row gather
    const int gtid = threadIdx.x - 192;
    {  // zero this CTA's slice of the accumulator, then count the CTA on sync[0]
      const int per = (nacc + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x);
      const int lo = static_cast<int>(blockIdx.x) * per;
      const int hi = min(nacc, lo + per);
      for (int e = lo + gtid; e < hi; e += 128) args.acc[e] = 0.0f;
      gather_sync();
      if (gtid == 0) ptx::red_release_gpu_add(args.sync, 1);
    }
    constexpr int kRowsPerThread = TOK / 16;
    const int chunk = gtid & 7;
    const int r0 = gtid >> 3;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int arrived = 0;  // stages this thread has arrived on
    auto acquire = [&]() {
      if (!ptx::mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, args.wait_ns)) {
        fail();
        ok = false;
      }
      return ok;
    };
    auto advance = [&]() {
      ++arrived;
      if (++stage == C::kStages) {
        stage = 0;
        phase ^= 1u;
      }
    };
    for (int i = 0; ok && i <= n_my; ++i) {
      if (i < n_my) {
        const TileInfo t = tile_of(i);
        const int e_blk = t.shared_blk ? 0 : block_exp(t.blk);
        const uint16_t* src[kRowsPerThread];
        uint32_t nbytes[kRowsPerThread];
#pragma unroll
        for (int r = 0; r < kRowsPerThread; ++r) {
          const int row = r0 + 16 * r;
          int tok = 0;
          bool valid;
          if (!t.shared_blk) {
            const int slot = row_slot(t.blk, e_blk, row);
            valid = static_cast<unsigned>(slot) < static_cast<unsigned>(args.S);
            if (valid) tok = slot / args.k;
          } else {
            tok = (t.blk - routed_blocks) * args.block_m + row;
            valid = tok < args.T;
            if (!valid) tok = 0;
          }
          src[r] = args.x + static_cast<size_t>(tok) * args.d + chunk * 8;
          nbytes[r] = valid ? 16u : 0u;
        }
        for (int s = 0; s < ng && acquire(); ++s) {
          const int kb = s / C::kGU;  // SwiGLU: the gate and the up stage of a K block carry the same rows
          const uint32_t sX = ptx::smem_u32(smem + stage * C::kStageBytes + C::kWBytes);
#pragma unroll
          for (int r = 0; r < kRowsPerThread; ++r) {
            const int row = r0 + 16 * r;
            const uint32_t dst = sX + (row >> 3) * 1024 + (row & 7) * 128 + ((chunk ^ (row & 7)) << 4);
            ptx::cp_async_16(dst, src[r] + kb * 64, nbytes[r]);
          }
          ptx::cp_async_arrive_noinc(&full[stage]);
          advance();
        }
      }
      if (ok && i >= 1) {
        for (int s = 0; s < nk2 && acquire(); ++s) {
          ptx::mbar_arrive(&full[stage]);  // down-GEMM stages carry weights only
          advance();
        }
      }
    }
    cp_async_wait_all();
    if constexpr (!FP8) {
      // after an abort: arrive on every stage the producer filled and this
      // thread did not, so that the producer can wait for its own loads
      exit_handshake();
      for (const int target = *prod_issued; arrived < target;) {
        ptx::mbar_arrive(&full[stage]);
        advance();
      }
      exit_handshake();
    }
  } else if constexpr (FP8) {
    // ------------------------------------------------ fp8 weights -> bf16 operand stages
    // Every stage of this CTA (the producer's order): wait for the raw
    // stage's bytes and for the operand stage to be free, expand the 128 x 64
    // e4m3 values times their power-of-two scales into bf16 (exact: an e4m3
    // value has 4 significant bits) in the 128-byte-swizzled K-major layout
    // the tensor core reads, and hand both stages on.  Thread: rows
    // r0 + 32 j (j < 4) of the stage, 16 K values each (q-th quarter).
    const int ctid = static_cast<int>(threadIdx.x) - 320;
    const int q = ctid & 3;
    const int r0 = ctid >> 2;
    int stage = 0, rstage = 0;
    uint32_t phase = 0, rphase = 0;
    const int total = n_my * (ng + nk2);
    for (int st = 0; st < total; ++st) {
      if (!ptx::mbar_wait_bounded(&raw_full[rstage], rphase, abort_flag, args.wait_ns) ||
          !ptx::mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, args.wait_ns)) {
        fail();
        break;
      }
      const uint8_t* rb = raw + rstage * C::kRawStageBytes;
      uint8_t* sW = smem + stage * C::kStageBytes;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = r0 + 32 * j;
        const uint4 v = *reinterpret_cast<const uint4*>(rb + r * 64 + q * 16);
        // scale byte b (1..254): 2^(b - 127), an fp32 with that exponent field
        const float scale = __uint_as_float(static_cast<uint32_t>(rb[C::kRawWBytes + (q >> 1) * 128 + r]) << 23);
        uint4 lo, hi;
        lo.x = e4m3x2_to_bf16x2(v.x & 0xFFFFu, scale);
        lo.y = e4m3x2_to_bf16x2(v.x >> 16, scale);
        lo.z = e4m3x2_to_bf16x2(v.y & 0xFFFFu, scale);
        lo.w = e4m3x2_to_bf16x2(v.y >> 16, scale);
        hi.x = e4m3x2_to_bf16x2(v.z & 0xFFFFu, scale);
        hi.y = e4m3x2_to_bf16x2(v.z >> 16, scale);
        hi.z = e4m3x2_to_bf16x2(v.w & 0xFFFFu, scale);
        hi.w = e4m3x2_to_bf16x2(v.w >> 16, scale);
        uint8_t* row = sW + (r >> 3) * 1024 + (r & 7) * 128;
        *reinterpret_cast<uint4*>(row + (((2 * q) ^ (r & 7)) << 4)) = lo;
        *reinterpret_cast<uint4*>(row + (((2 * q + 1) ^ (r & 7)) << 4)) = hi;
      }
      ptx::fence_proxy_async_smem();  // the tensor core reads these rows next
      ptx::mbar_arrive(&full[stage]);
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&raw_empty[rstage]);
      if (++stage == C::kStages) {
        stage = 0;
        phase ^= 1u;
      }
      if (++rstage == C::kRawStages) {
        rstage = 0;
        rphase ^= 1u;
      }
    }
  }

  // every warp reconverges (the idle lanes of the producer and MMA warps
  // wait for their working lane) before the block-wide barrier
  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  // ---- grid end: all reductions issued -> convert the accumulator to bf16.
  // sync[1] counts the CTAs that have issued all their reductions; the last
  // one to arrive returns sync[0] and sync[1] to zero.  A small output is
  // then converted by that CTA alone while the others leave.  Otherwise the
  // last CTA releases the others by moving the generation in sync[2] on by
  // one (each CTA read it before counting itself, and waits for it to
  // change) and every CTA converts its slice.  A CTA that gave up (a wait
  // ran out) counts itself and leaves; since nothing is handed back, the
  // counters are consistent for the next launch whichever CTAs gave up.
  const bool last_converts = nacc <= kLastCtaConvertMax;
  if (threadIdx.x == 0) {
    const int G = static_cast<int>(gridDim.x);
    const bool aborted = *abort_flag != 0;  // final: every role has finished
    // the last CTA moves the generation on only after this CTA's count below
    const int gen = ptx::ld_acquire_gpu(args.sync + 2);
    int mode = 0;  // 0: leave, 1: convert this CTA's slice, 2: convert everything
    if (ptx::atom_acq_rel_gpu_add(args.sync + 1, 1) == G - 1) {  // releases this CTA's reductions
      args.sync[0] = 0;
      args.sync[1] = 0;
      if (last_converts) {
        mode = 2;
      } else {
        ptx::st_release_gpu(args.sync + 2, static_cast<int>(static_cast<uint32_t>(gen) + 1u));
        mode = 1;
      }
    } else if (!last_converts && !aborted) {
      if (spin_until_changed(args.sync + 2, gen, args.wait_ns))
        mode = 1;
      else
        fail();
    }
    *flag = mode;
  }
  if (warp == 1) {  // TMEM is freed while thread 0 waits at the grid barrier
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, 512);
  }
  __syncthreads();
  if (*flag) {
    const int per = ((nacc + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x) + 3) & ~3;
    const int lo = *flag == 2 ? 0 : static_cast<int>(blockIdx.x) * per;
    const int hi = *flag == 2 ? nacc : min(nacc, lo + per);
    const bool vec = (reinterpret_cast<uintptr_t>(args.out) & 7) == 0;
#pragma unroll 4
    for (int e = lo + 4 * static_cast<int>(threadIdx.x); e < hi; e += 4 * C::kNumThreads) {
      if (vec && e + 4 <= hi) {
        const float4 a = __ldcg(reinterpret_cast<const float4*>(args.acc + e));
        uint2 o;
        o.x = pack_bf16x2(a.x, a.y);
        o.y = pack_bf16x2(a.z, a.w);
        *reinterpret_cast<uint2*>(args.out + e) = o;
      } else {
        for (int m = e; m < min(hi, e + 4); ++m) args.out[m] = float_to_bf16_bits(__ldcg(args.acc + m));
      }
    }
  }
}

template <int EPI1, int TOK, bool ROUTE, bool FP8 = false>
cudaError_t launch_fused_variant(const FusedArgs& args, int grid, cudaStream_t stream) {
  using C = FusedCfg<EPI1, TOK, ROUTE, FP8>;
  auto kern = fused_expert_kernel<EPI1, TOK, ROUTE, FP8>;
  // per device, set once; concurrent first calls may both set it (idempotent)
  static std::atomic<bool> attr_done[64];
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_done[dev].load(std::memory_order_acquire)) {
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (err != cudaSuccess) return err;
    attr_done[dev].store(true, std::memory_order_release);
  }
  return launch_pdl(kern, dim3(grid), dim3(C::kNumThreads), C::kSmemBytes, stream, args);
}

}  // namespace

bool fused_expert_supported(int block_m) { return block_m == 16 || block_m == 32 || block_m == 64; }

int64_t fused_expert_max_tiles(int act_epi, int total_blocks_max, int F) {
  (void)act_epi;  // 128 h columns per tile for both activations
  return static_cast<int64_t>(total_blocks_max) * ((F + 127) / 128);
}

bool fused_routing_supported(int T, int k, int E, int n_group, int block_m) {
  return block_m == 16 && static_cast<int64_t>(T) * k <= kRouteMaxS && E <= MOE_MAX_EXPERTS && n_group <= 64;
}

cudaError_t launch_fused_expert(int act_epi, int block_m, bool route, const FusedArgs& args, int grid,
                                cudaStream_t stream, bool fp8) {
  const bool gated = act_epi == kEpiSwiGLU;
  if (fp8) {
    if (route) {
      if (block_m != 16) return cudaErrorInvalidValue;
      return gated ? launch_fused_variant<kEpiSwiGLU, 16, true, true>(args, grid, stream)
                   : launch_fused_variant<kEpiRelu2, 16, true, true>(args, grid, stream);
    }
    switch (block_m) {
      case 16:
        return gated ? launch_fused_variant<kEpiSwiGLU, 16, false, true>(args, grid, stream)
                     : launch_fused_variant<kEpiRelu2, 16, false, true>(args, grid, stream);
      case 32:
        return gated ? launch_fused_variant<kEpiSwiGLU, 32, false, true>(args, grid, stream)
                     : launch_fused_variant<kEpiRelu2, 32, false, true>(args, grid, stream);
      case 64:
        return gated ? launch_fused_variant<kEpiSwiGLU, 64, false, true>(args, grid, stream)
                     : launch_fused_variant<kEpiRelu2, 64, false, true>(args, grid, stream);
      default:
        return cudaErrorInvalidValue;
    }
  }
  if (route) {
    if (block_m != 16) return cudaErrorInvalidValue;
    return gated ? launch_fused_variant<kEpiSwiGLU, 16, true>(args, grid, stream)
                 : launch_fused_variant<kEpiRelu2, 16, true>(args, grid, stream);
  }
  switch (block_m) {
    case 16:
      return gated ? launch_fused_variant<kEpiSwiGLU, 16, false>(args, grid, stream)
                   : launch_fused_variant<kEpiRelu2, 16, false>(args, grid, stream);
    case 32:
      return gated ? launch_fused_variant<kEpiSwiGLU, 32, false>(args, grid, stream)
                   : launch_fused_variant<kEpiRelu2, 32, false>(args, grid, stream);
    case 64:
      return gated ? launch_fused_variant<kEpiSwiGLU, 64, false>(args, grid, stream)
                   : launch_fused_variant<kEpiRelu2, 64, false>(args, grid, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace moe
