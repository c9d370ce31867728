// Token-major grouped GEMMs on CTA pairs (tcgen05 cta_group::2).
//
// The same computations as grouped_gemm.cu -- the "Grouped GEMM Structure"
// of the fused-moe-kernel page ("Fused MoE Kernel Optimization", skillmd
// zjli2013): the gate/up GEMM with `act_fn(gate) * up` (or the relu^2 fc1 of
// the mlxcel PR) written as h, and the down GEMM whose rows, scaled by their
// top-k weight, are added into the fp32 [T, d] accumulator at their token
// ("Common Pitfalls" 4; the weighted sum of the axolotl
// `_moe_triton_forward`, src/axolotl/monkeypatch/deepseek_v3/__init__.py) --
// with a 256 x 256 tile per pair of SMs instead of 128 x 256 per SM.  Both
// operands arrive by TMA: the gate/up GEMM reads its token rows from a copy
// of x already permuted into the expert-sorted row order (permute.cu).
//
// A cluster of two CTAs works on a "pair unit": two consecutive 128-row
// blocks of the same expert (the last block of an expert with an odd count
// is paired with nothing; the odd CTA then computes rows it discards).  Each
// CTA loads its own block's token rows (A: permuted x or h) and half of the
// 256 weight rows of the tile (B; SwiGLU: the even CTA the 128 gate rows,
// the odd CTA the matching 128 up rows) by TMA; the transaction bytes of both CTAs complete on the even
// CTA's full barrier, where its single MMA thread issues M = 256, N = 256
// MMAs that read A and B from both CTAs' shared memory.  Commits go to both
// CTAs (empty stages, full accumulators).  Each CTA's epilogue drains its own
// TMEM half (its 128 rows) and signals the even CTA that the accumulator is
// free.  Per SM and 64-wide K step the pair moves 32 KB of operands instead
// of 48 KB, so the same shared memory holds six stages instead of four.
//
// Every mbarrier wait is bounded; on expiry the CTA records
// MOE_ERR_DEVICE_TIMEOUT and its roles leave their loops; the even CTA then
// waits for its MMAs and for its stages' loads still in flight.  Both CTAs
// always reach the closing cluster barrier, which orders the peer's last
// remote arrivals before either CTA frees its TMEM and exits.
#include <atomic>
#include "common.cuh"
#include "gemm.h"
#include "ptx.cuh"

namespace moe {

namespace {

// After an abort, the odd CTA's wait for its last loads to land (they
// complete on the even CTA's barriers): far above a TMA load's latency.
constexpr uint64_t kDrainGraceNs = 50000;

template <int EPI>
struct PairCfg {
  static constexpr bool kGated = EPI == kEpiSwiGLU;
  static constexpr bool kZero = EPI != kEpiScale;  // gate/up: a warp zeroes the down GEMM's accumulator
  static constexpr int kOutCols = kGated ? 128 : 256;  // output columns of a tile
  static constexpr int kABytes = 128 * 128;  // 128 token rows x 64 bf16
  static constexpr int kBBytes = 128 * 128;  // 128 weight rows x 64 bf16 (this CTA's half of N = 256)
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = 6;
  static constexpr int kAccCols = 256;
  static constexpr int kTmemCols = 512;
  static constexpr int kNumThreads = kZero ? 224 : 192;  // producer, MMA, 4 epilogue warps (+ zeroing)
  static constexpr int kBarrierBytes = 256;
  static constexpr int kRedStride = 33;
  static constexpr int kRedBytes = kZero ? 0 : 4 * 32 * kRedStride * 4;
  static constexpr int kMaxUnits = 2048;  // pair units of one launch
  static constexpr int kUnitBytes = kMaxUnits * 4;
  static constexpr int kSmemBytes = kStages * kStageBytes + kBarrierBytes + kRedBytes + kUnitBytes + 1024;
  static constexpr uint32_t kIdesc = ptx::idesc_bf16_f32(256, 256);
  static_assert((2 * kStages + 5) * 8 + 16 <= kBarrierBytes, "barrier area");
  static_assert(kSmemBytes <= 232448, "shared memory per block");
};

// silu(g) = g * sigmoid(g), with the fast approximate divide: h is rounded
// to bf16 right after, far coarser than the divide's error.
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

__device__ __forceinline__ void red_add_v4_f32(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

struct PairTile {
  int b0;      // first block of the unit
  int nb;      // blocks in the unit (1 or 2)
  int wt;      // 256-wide output column tile
  bool shared_blk;
};

template <int EPI>
__global__ void __launch_bounds__(PairCfg<EPI>::kNumThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ GemmArgs args) {
  using C = PairCfg<EPI>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;  // even CTA: the MMA issuer's last commit (drain before TMEM is freed)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* never = reinterpret_cast<volatile int*>(tmem_holder + 3);  // stays 0: drains ignore the abort
  float* red_buf = reinterpret_cast<float*>(smem + C::kStages * C::kStageBytes + C::kBarrierBytes);
  int* unit_b0 = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(red_buf) + C::kRedBytes);

  const int warp = threadIdx.x / kWarp;
  const int lane = threadIdx.x % kWarp;
  const uint32_t rank = ptx::cluster_ctarank();  // 0: issues the pair's MMAs
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      ptx::mbar_init(&full[s], 1);   // even CTA: its producer's arrive + both CTAs' bytes
      ptx::mbar_init(&empty[s], 1);  // one commit of the pair's MMA
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&tfull[b], 1 + args.tfull_surplus);
      ptx::mbar_init(&tempty[b], 8);  // even CTA: four epilogue warps of each CTA
    }
    ptx::mbar_init(mma_done, 1);
    *abort_flag = 0;
    *never = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&args.tm_w);
    if (args.n_shared_blocks) ptx::prefetch_tmap(&args.tm_ws);
    ptx::prefetch_tmap(&args.tm_x);
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(tmem_holder, C::kTmemCols);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // both CTAs' barriers exist before any remote arrival
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  pdl_wait();
  pdl_launch_dependents();
  int routed_blocks = *args.ntpp / args.block_m;
  if (routed_blocks < 0) routed_blocks = 0;
  if (routed_blocks > args.max_routed_blocks) routed_blocks = args.max_routed_blocks;
  const int total_blocks = routed_blocks + args.n_shared_blocks;

  // ---- pair units: a unit starts at the first block of an expert's run and
  // at every second block after it (the shared expert's blocks are one run)
  if (warp == 0) {
    int seg_start = 0, n_units = 0, prev_e = -2;
    for (int base = 0; base < total_blocks; base += kWarp) {
      const int b = base + lane;
      int e = -3;
      if (b < total_blocks) e = b < routed_blocks ? args.expert_ids[b] : -1;
      const int pe = __shfl_up_sync(0xffffffffu, e, 1);
      const int left = lane == 0 ? prev_e : pe;
      const bool new_seg = b < total_blocks && (b == 0 || e != left);
      const unsigned segs = __ballot_sync(0xffffffffu, new_seg);
      const unsigned upto = segs & (0xffffffffu >> (31 - lane));
      const int my_seg = upto ? base + (31 - __clz(upto)) : seg_start;
      const bool start = b < total_blocks && ((b - my_seg) & 1) == 0;
      const unsigned starts = __ballot_sync(0xffffffffu, start);
      const int idx = n_units + __popc(starts & ((1u << lane) - 1u));
      if (start && idx < C::kMaxUnits) unit_b0[idx] = b;
      n_units += __popc(starts);
      seg_start = __shfl_sync(0xffffffffu, my_seg, 31);
      prev_e = __shfl_sync(0xffffffffu, e, 31);
    }
    if (lane == 0) tmem_holder[2] = static_cast<uint32_t>(n_units < C::kMaxUnits ? n_units : C::kMaxUnits);
  }
  __syncthreads();
  const int n_units = static_cast<int>(tmem_holder[2]);
  const int n_wt = (args.n_out + C::kOutCols - 1) / C::kOutCols;
  const int pass_w = args.pass_cols > 0 && args.pass_cols < n_wt ? args.pass_cols : n_wt;
  const int total_tiles = n_units * n_wt;
  const int nk = args.K / 64;

  auto tile_of = [&](int tile) {
    const int per_pass = n_units * pass_w;
    const int ps = tile / per_pass;
    const int w0 = ps * pass_w;
    const int width = n_wt - w0 < pass_w ? n_wt - w0 : pass_w;
    const int r = tile - ps * per_pass;
    const int u = r / width;
    PairTile t;
    t.b0 = unit_b0[u];
    const int next = u + 1 < n_units ? unit_b0[u + 1] : total_blocks;
    t.nb = next - t.b0 >= 2 ? 2 : 1;
    t.wt = w0 + (r - u * width);
    t.shared_blk = t.b0 >= routed_blocks;
    return t;
  };
  auto fail = [&]() {
    *abort_flag = 1;
    set_status(args.status, MOE_ERR_DEVICE_TIMEOUT);
  };

  if (warp == 0) {
    // ------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int issued = 0;  // stages filled so far
      for (int tile = pair; ok && tile < total_tiles; tile += n_pairs) {
        const PairTile t = tile_of(tile);
        const CUtensorMap* tm = t.shared_blk ? &args.tm_ws : &args.tm_w;
        int e = 0;
        if (!t.shared_blk) {
          e = args.expert_ids[t.b0];
          if (e < 0 || e >= args.E) set_status(args.status, MOE_ERR_BAD_EXPERT_ID);
        }
        // this CTA's block (the odd CTA of a one-block unit loads the even
        // CTA's rows again and discards its result)
        const int blk = t.b0 + (static_cast<int>(rank) < t.nb ? static_cast<int>(rank) : 0);
        const int wrow = C::kGated ? t.wt * 128 + (rank ? args.up_row_offset : 0)
                                   : t.wt * 256 + static_cast<int>(rank) * 128;
        for (int kb = 0; kb < nk; ++kb) {
          if (!ptx::mbar_wait_cluster_bounded(&empty[stage], phase ^ 1u, abort_flag, args.wait_ns)) {
            fail();
            ok = false;
            break;
          }
          uint8_t* sA = smem + stage * C::kStageBytes;
          if (rank == 0) ptx::mbar_arrive_expect_tx(&full[stage], 2 * C::kStageBytes);
          ptx::tma_load_2d_pair(sA, &args.tm_x, &full[stage], kb * 64, blk * args.block_m);
          ptx::tma_load_3d_pair(sA + C::kABytes, tm, &full[stage], kb * 64, wrow, e);
          ++issued;
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // The even CTA's full barriers count both CTAs' bytes: before the pair
      // releases its shared memory, the even CTA waits for the last phase of
      // every stage it filled (at once after a normal run).  The odd CTA's
      // loads complete only on the even CTA's barriers, which it cannot wait
      // on; after an abort it may have filled a phase the even CTA never
      // did, so it then gives its last loads a fixed grace period to land.
      if (rank != 0 && !ok) {
        const uint64_t t0 = ptx::globaltimer_ns();
        while (ptx::globaltimer_ns() - t0 < kDrainGraceNs) __nanosleep(256);
      }
      if (rank == 0) {
        for (int j = 1; j <= C::kStages && j <= issued; ++j) {
          int st = stage - j;
          uint32_t ph = phase;
          if (st < 0) {
            st += C::kStages;
            ph ^= 1u;
          }
          ptx::mbar_wait_cluster_bounded(&full[st], ph, never, kDrainLimitNs);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int abuf = 0;
      uint32_t aphase = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total_tiles; tile += n_pairs) {
        if (!ptx::mbar_wait_cluster_bounded(&tempty[abuf], aphase ^ 1u, abort_flag, args.wait_ns)) {
          fail();
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(abuf * C::kAccCols);
        for (int kb = 0; kb < nk; ++kb) {
          if (!ptx::mbar_wait_cluster_bounded(&full[stage], phase, abort_flag, args.wait_ns)) {
            fail();
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t sA = ptx::smem_u32(smem + stage * C::kStageBytes);
          const uint32_t sB = sA + C::kABytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::mma_bf16_pair(d_tmem, ptx::sw128_kmajor_desc(sA + kk * 32), ptx::sw128_kmajor_desc(sB + kk * 32),
                               C::kIdesc, (kb | kk) != 0 ? 1u : 0u);
          ptx::mma_commit_pair(&empty[stage]);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        ptx::mma_commit_pair(&tfull[abuf]);
        if (++abuf == 2) {
          abuf = 0;
          aphase ^= 1u;
        }
      }
      // no MMA of the pair may still run when TMEM is freed: the last commit
      // arrives on both CTAs' mma_done (every tcgen05 operation of the kernel
      // is a cta_group::2 one)
      ptx::mma_commit_pair(mma_done);
      if (!ptx::mbar_wait_bounded(mma_done, 0u, never, kDrainLimitNs)) fail();
    } else if (lane == 0) {
      // odd CTA: the even CTA's final commit also arrives here
      if (!ptx::mbar_wait_cluster_bounded(mma_done, 0u, never, kDrainLimitNs)) fail();
    }
  } else if (warp < 6) {
    // ------------------------------------------------ epilogue (both CTAs, own TMEM half)
    const int q = warp & 3;
    const int row = q * 32 + lane;
    float* stg = red_buf + q * 32 * C::kRedStride;
    const int rr = lane >> 3;
    const int cc = (lane & 7) * 4;
    int abuf = 0;
    uint32_t aphase = 0;
    for (int tile = pair; tile < total_tiles; tile += n_pairs) {
      const PairTile t = tile_of(tile);
      if (!ptx::mbar_wait_cluster_bounded(&tfull[abuf], aphase, abort_flag, args.wait_ns)) {
        fail();
        break;
      }
      ptx::tc_fence_after();
      const uint32_t t_acc =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(abuf * C::kAccCols);
      if (static_cast<int>(rank) < t.nb && EPI == kEpiSwiGLU) {
        const int p = (t.b0 + static_cast<int>(rank)) * args.block_m + row;
        uint16_t* orow = static_cast<uint16_t*>(args.out) + static_cast<size_t>(p) * args.n_out;
        // 32 h columns per TMEM wait (F is a multiple of 64, so a chunk is
        // either wholly inside the layer or wholly past it)
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t g[32], u[32];
          ptx::tmem_ld16(t_acc + c0, *reinterpret_cast<uint32_t(*)[16]>(&g[0]));
          ptx::tmem_ld16(t_acc + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&g[16]));
          ptx::tmem_ld16(t_acc + 128 + c0, *reinterpret_cast<uint32_t(*)[16]>(&u[0]));
          ptx::tmem_ld16(t_acc + 128 + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&u[16]));
          ptx::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) asm volatile("" : "+r"(g[j]), "+r"(u[j]));  // uses stay after the wait
          const int col = t.wt * 128 + c0;
          if (col < args.n_out) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float h0 = silu_f(__uint_as_float(g[2 * i])) * __uint_as_float(u[2 * i]);
              const float h1 = silu_f(__uint_as_float(g[2 * i + 1])) * __uint_as_float(u[2 * i + 1]);
              pk[i] = pack_bf16x2(h0, h1);
            }
            uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
      } else if (static_cast<int>(rank) < t.nb && EPI == kEpiRelu2) {
        const int p = (t.b0 + static_cast<int>(rank)) * args.block_m + row;
        uint16_t* orow = static_cast<uint16_t*>(args.out) + static_cast<size_t>(p) * args.n_out;
#pragma unroll 1
        for (int c0 = 0; c0 < 256; c0 += 16) {
          uint32_t a[16];
          ptx::tmem_ld16(t_acc + c0, a);
          ptx::tmem_wait_ld();
          const int col = t.wt * 256 + c0;
          if (col < args.n_out) {
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float v0 = fmaxf(__uint_as_float(a[2 * i]), 0.0f);
              const float v1 = fmaxf(__uint_as_float(a[2 * i + 1]), 0.0f);
              pk[i] = pack_bf16x2(v0 * v0, v1 * v1);
            }
            uint4* dst = reinterpret_cast<uint4*>(orow + col);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      } else if (static_cast<int>(rank) < t.nb) {
        const int blk = t.b0 + static_cast<int>(rank);
        const int p = blk * args.block_m + row;
        bool valid;
        int tok;
        float wrow = 1.0f;
        if (blk < routed_blocks) {
          const int slot = args.sorted_ids[p];
          valid = static_cast<unsigned>(slot) < static_cast<unsigned>(args.S);
          tok = valid ? slot / args.k : 0;
          if (valid) wrow = args.topk_w[slot];
        } else {
          tok = (blk - routed_blocks) * args.block_m + row;
          valid = tok < args.T;
        }
#pragma unroll 1
        for (int c0 = 0; c0 < 256; c0 += 32) {
          uint32_t a[32];
          ptx::tmem_ld16(t_acc + c0, *reinterpret_cast<uint32_t(*)[16]>(&a[0]));
          ptx::tmem_ld16(t_acc + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&a[16]));
          ptx::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) asm volatile("" : "+r"(a[j]));  // uses stay after the wait
          const int col = t.wt * 256 + c0;
          if (col >= args.n_out) break;  // uniform across the warp
#pragma unroll
          for (int j = 0; j < 32; ++j) stg[lane * C::kRedStride + j] = __uint_as_float(a[j]) * wrow;
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = 4 * i + rr;
            const int tk = __shfl_sync(0xffffffffu, tok, r);
            const int ok = __shfl_sync(0xffffffffu, valid ? 1 : 0, r);
            const float* src = stg + r * C::kRedStride + cc;
            if (ok)
              red_add_v4_f32(args.acc + static_cast<size_t>(tk) * args.n_out + col + cc, src[0], src[1], src[2],
                             src[3]);
          }
          __syncwarp();
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_leader(&tempty[abuf]);
      if (++abuf == 2) {
        abuf = 0;
        aphase ^= 1u;
      }
    }
  } else if (C::kZero) {
    // ------------------------------------------------ zero this CTA's share of the down GEMM's accumulator
    if (args.acc != nullptr) {
      const int64_t n = args.acc_elems;
      const int64_t per = ((n + gridDim.x - 1) / gridDim.x + 3) & ~int64_t(3);
      const int64_t lo = static_cast<int64_t>(blockIdx.x) * per;
      const int64_t hi = lo + per < n ? lo + per : n;
      for (int64_t i = lo + 4 * lane; i < hi; i += 4 * kWarp) {
        if (i + 4 <= hi)
          *reinterpret_cast<float4*>(args.acc + i) = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        else
          for (int64_t m = i; m < hi; ++m) args.acc[m] = 0.0f;
      }
    }
  }

  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // the peer's last arrivals and reads are done
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem_base, C::kTmemCols);
  }
}

template <int EPI>
cudaError_t launch_pair_variant(const GemmArgs& args, int grid, cudaStream_t stream) {
  using C = PairCfg<EPI>;
  auto kern = grouped_gemm_pair_kernel<EPI>;
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
  grid &= ~1;
  if (grid < 2) grid = 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(C::kNumThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, args);
}

}  // namespace

bool gemm_pair_supported(int block_m, int total_blocks_max) {
  return block_m == 128 && total_blocks_max <= PairCfg<kEpiScale>::kMaxUnits;
}

cudaError_t launch_grouped_gemm_pair(int epi, const GemmArgs& args, int grid, cudaStream_t stream) {
  if (args.block_m != 128) return cudaErrorInvalidValue;
  switch (epi) {
    case kEpiSwiGLU: return launch_pair_variant<kEpiSwiGLU>(args, grid, stream);
    case kEpiRelu2: return launch_pair_variant<kEpiRelu2>(args, grid, stream);
    case kEpiScale: return launch_pair_variant<kEpiScale>(args, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace moe
