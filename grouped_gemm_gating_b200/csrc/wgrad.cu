// Per-expert weight gradients of the MoE layer's backward on the
// 5th-generation tensor cores (tcgen05), sm_100a.
//
// The axolotl vendor-moe diff's grouped backward
// (src/axolotl/kernels/moe/tt_cg_gemm/cg_backward.py, `_kernel_cg_backward_dw`)
// computes each expert's weight gradient as a sum over the rows routed to
// that expert.  Here, with the rows in the expert-sorted order of the forward
// (sorted_token_ids / expert_ids, each expert's run padded to 128 rows with
// zero rows):
//
//   dW13_e = da_e^T x_e     (M = n1 rows of W13, N = d,  K = the expert's rows)
//   dW2_e  = dout_e^T (w h)_e (M = d,            N = F,  K = the expert's rows)
//
// The reduction runs over rows, so both operands are read with their output
// index contiguous (MN-major): TMA boxes of {64 M (or N) values, 64 rows}
// with 128-byte swizzle land in the canonical MN-major layout, two such boxes
// side by side for the 128 M values of a tile and four for its 256 N values.
//
// Tiles are (expert, 128-row M tile, 256-column N tile); every CTA finds the
// experts' block runs from expert_ids and walks the tiles with the largest
// experts first (a static stride over that order balances experts whose row
// counts differ by orders of magnitude).  An expert with no rows gets zero
// tiles written.  Warp roles: warp 0 TMA producer, warp 1 TMEM allocator and
// MMA issuer, warps 2-5 epilogue (TMEM -> bf16 -> global, one TMEM lane
// quadrant each).  Every wait is bounded; after giving up the producer waits
// for its own loads and the MMA issuer for its MMAs before TMEM is freed.
#include <atomic>

#include "common.cuh"
#include "gemm.h"
#include "ptx.cuh"

namespace moe {

namespace {

struct WgCfg {
  static constexpr int kABytes = 2 * 8192;  // 128 M values x 64 rows
  static constexpr int kBBytes = 4 * 8192;  // 256 N values x 64 rows
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = 4;
  static constexpr int kAccCols = 256;
  static constexpr int kTmemCols = 512;
  static constexpr int kNumThreads = 192;
  static constexpr int kMaxSeg = MOE_MAX_EXPERTS + 1;  // routed experts + the shared one
  static constexpr int kBarrierBytes = 256;
  static constexpr int kSegBytes = 3 * kMaxSeg * 4;     // block count, first block, order
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024 + kBarrierBytes + kSegBytes;
  static constexpr uint32_t kIdesc = ptx::idesc_bf16_f32(128, 256, true, true);
  static_assert((2 * kStages + 5) * 8 + 16 <= kBarrierBytes, "barrier area");
  static_assert(kSmemBytes <= 232448, "shared memory per block");
};

__global__ void __launch_bounds__(WgCfg::kNumThreads, 1) wgrad_kernel(const __grid_constant__ WgradArgs args) {
  using C = WgCfg;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* never = reinterpret_cast<volatile int*>(tmem_holder + 2);
  int* seg_cnt = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(full) + C::kBarrierBytes);
  int* seg_first = seg_cnt + C::kMaxSeg;
  int* order = seg_first + C::kMaxSeg;

  const int warp = threadIdx.x / kWarp;
  const int lane = threadIdx.x % kWarp;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&tfull[b], 1);
      ptx::mbar_init(&tempty[b], 4);
    }
    ptx::mbar_init(mma_done, 1);
    *abort_flag = 0;
    *never = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&args.tm_a);
    ptx::prefetch_tmap(&args.tm_b);
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_holder, C::kTmemCols);
    ptx::tmem_relinquish();
  }
  const int E_tot = args.E + (args.n_shared_blocks > 0 ? 1 : 0);
  for (int e = threadIdx.x; e < C::kMaxSeg; e += C::kNumThreads) {
    seg_cnt[e] = 0;
    seg_first[e] = 0x7fffffff;
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  pdl_wait();
  pdl_launch_dependents();
  int routed_blocks = *args.ntpp / args.block_m;
  if (routed_blocks < 0) routed_blocks = 0;
  if (routed_blocks > args.max_routed_blocks) routed_blocks = args.max_routed_blocks;
  // ---- each expert's run of blocks (blocks are sorted by expert)
  for (int b = threadIdx.x; b < routed_blocks; b += C::kNumThreads) {
    const int e = args.expert_ids[b];
    if (e < 0 || e >= args.E) {
      set_status(args.status, MOE_ERR_BAD_EXPERT_ID);
      continue;
    }
    atomicAdd(&seg_cnt[e], 1);
    atomicMin(&seg_first[e], b);
  }
  if (threadIdx.x == 0 && args.n_shared_blocks > 0) {
    seg_cnt[args.E] = args.n_shared_blocks;
    seg_first[args.E] = routed_blocks;
  }
  __syncthreads();
  // ---- largest experts first: order[rank] = e, ranked by (blocks desc, id asc)
  for (int e = threadIdx.x; e < E_tot; e += C::kNumThreads) {
    const int c = seg_cnt[e];
    int rank = 0;
    for (int f = 0; f < E_tot; ++f) {
      const int cf = seg_cnt[f];
      rank += (cf > c || (cf == c && f < e)) ? 1 : 0;
    }
    order[rank] = e;
  }
  __syncthreads();

  const int n_mt = (args.M + 127) / 128;
  const int n_nt = (args.N + 255) / 256;
  const int per_e = n_mt * n_nt;
  const int total_tiles = E_tot * per_e;
  auto fail = [&]() {
    *abort_flag = 1;
    set_status(args.status, MOE_ERR_DEVICE_TIMEOUT);
  };
  struct Tile {
    int e, mt, nt, cnt, first;
  };
  auto tile_of = [&](int t) {
    Tile r;
    const int i = t / per_e;
    const int w = t - i * per_e;
    r.e = order[i];
    r.mt = w / n_nt;
    r.nt = w - r.mt * n_nt;
    r.cnt = seg_cnt[r.e];
    r.first = seg_first[r.e];
    return r;
  };

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int issued = 0;
      for (int t = blockIdx.x; ok && t < total_tiles; t += gridDim.x) {
        const Tile tl = tile_of(t);
        const int nk = tl.cnt * (args.block_m / 64);
        for (int ks = 0; ks < nk; ++ks) {
          if (!ptx::mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, args.wait_ns)) {
            fail();
            ok = false;
            break;
          }
          const int row = tl.first * args.block_m + ks * 64;
          uint8_t* sA = smem + stage * C::kStageBytes;
          uint8_t* sB = sA + C::kABytes;
          ptx::mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
#pragma unroll
          for (int j = 0; j < 2; ++j) ptx::tma_load_2d(sA + j * 8192, &args.tm_a, &full[stage], tl.mt * 128 + 64 * j, row);
#pragma unroll
          for (int j = 0; j < 4; ++j) ptx::tma_load_2d(sB + j * 8192, &args.tm_b, &full[stage], tl.nt * 256 + 64 * j, row);
          ++issued;
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // the last load into every stage lands before shared memory is released
      for (int j = 1; j <= C::kStages && j <= issued; ++j) {
        int st = stage - j;
        uint32_t ph = phase;
        if (st < 0) {
          st += C::kStages;
          ph ^= 1u;
        }
        ptx::mbar_wait_bounded(&full[st], ph, never, kDrainLimitNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int abuf = 0;
      uint32_t aphase = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < total_tiles; t += gridDim.x) {
        const Tile tl = tile_of(t);
        const int nk = tl.cnt * (args.block_m / 64);
        if (!ptx::mbar_wait_bounded(&tempty[abuf], aphase ^ 1u, abort_flag, args.wait_ns)) {
          fail();
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(abuf * C::kAccCols);
        for (int ks = 0; ks < nk; ++ks) {
          if (!ptx::mbar_wait_bounded(&full[stage], phase, abort_flag, args.wait_ns)) {
            fail();
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t sA = ptx::smem_u32(smem + stage * C::kStageBytes);
          const uint32_t sB = sA + C::kABytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::mma_bf16(d_tmem, ptx::sw128_mnmajor_desc(sA + kk * 2048, 8192),
                          ptx::sw128_mnmajor_desc(sB + kk * 2048, 8192), C::kIdesc, (ks | kk) != 0 ? 1u : 0u);
          ptx::mma_commit(&empty[stage]);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        ptx::mma_commit(&tfull[abuf]);  // with no rows: arrives at once, the epilogue writes zeros
        if (++abuf == 2) {
          abuf = 0;
          aphase ^= 1u;
        }
      }
      ptx::mma_commit(mma_done);
      if (!ptx::mbar_wait_bounded(mma_done, 0u, never, kDrainLimitNs)) fail();
    }
  } else {
    // ------------------------------------------------ epilogue: TMEM -> bf16 dW rows
    const int q = warp & 3;
    int abuf = 0;
    uint32_t aphase = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
      const Tile tl = tile_of(t);
      if (!ptx::mbar_wait_bounded(&tfull[abuf], aphase, abort_flag, args.wait_ns)) {
        fail();
        break;
      }
      ptx::tc_fence_after();
      const uint32_t t_acc =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(abuf * C::kAccCols);
      const int m = tl.mt * 128 + q * 32 + lane;
      uint16_t* base = tl.e < args.E ? args.out + static_cast<size_t>(tl.e) * args.M * args.N : args.out_shared;
      uint16_t* orow = base + static_cast<size_t>(m < args.M ? m : 0) * args.N;
#pragma unroll 1
      for (int c0 = 0; c0 < 256; c0 += 32) {
        const int col = tl.nt * 256 + c0;
        if (col >= args.N) break;  // uniform across the warp
        uint32_t a[32];
        if (tl.cnt > 0) {
          ptx::tmem_ld16(t_acc + c0, *reinterpret_cast<uint32_t(*)[16]>(&a[0]));
          ptx::tmem_ld16(t_acc + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&a[16]));
          ptx::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) asm volatile("" : "+r"(a[j]));  // uses stay after the wait
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) a[j] = 0u;
        }
        if (m < args.M) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(__uint_as_float(a[2 * i]), __uint_as_float(a[2 * i + 1]));
          uint4* dst = reinterpret_cast<uint4*>(orow + col);
          // N is a multiple of 64: a 32-column chunk is wholly inside or past it
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&tempty[abuf]);
      if (++abuf == 2) {
        abuf = 0;
        aphase ^= 1u;
      }
    }
  }

  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

}  // namespace

int64_t wgrad_max_tiles(int E, int n_shared, int M, int N) {
  return static_cast<int64_t>(E + (n_shared ? 1 : 0)) * ((M + 127) / 128) * ((N + 255) / 256);
}

cudaError_t launch_wgrad(const WgradArgs& args, int grid, cudaStream_t stream) {
  if (args.block_m != 128 || args.E + 1 > WgCfg::kMaxSeg || args.N % 64 != 0) return cudaErrorInvalidValue;
  auto kern = wgrad_kernel;
  static std::atomic<bool> attr_done[64];
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_done[dev].load(std::memory_order_acquire)) {
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, WgCfg::kSmemBytes);
    if (err != cudaSuccess) return err;
    attr_done[dev].store(true, std::memory_order_release);
  }
  return launch_pdl(kern, dim3(grid), dim3(WgCfg::kNumThreads), WgCfg::kSmemBytes, stream, args);
}

}  // namespace moe
