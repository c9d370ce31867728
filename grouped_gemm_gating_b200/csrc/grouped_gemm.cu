// Persistent, warp-specialised grouped GEMM on the 5th-generation tensor
// cores (tcgen05) of sm_100a, with the MoE epilogues fused in.
//
// This is the "Grouped GEMM Structure" of the fused-moe-kernel page ("Fused
// MoE Kernel Optimization", skillmd zjli2013): a tiled GEMM with an extra
// indirection, where sorted_token_ids maps each block of block_m rows to
// token rows, expert_ids maps the block to the expert whose [N, K] weight
// slice is used, and blocks at or past num_tokens_post_padded do no work.
// The gate/up projections and `act_fn(gate) * up` of the axolotl
// `_moe_triton_forward` (src/axolotl/monkeypatch/deepseek_v3/__init__.py) are
// one GEMM here with the activation in the epilogue; the squared-ReLU fc1 of
// the mlxcel PR ("fc1 -> relu^2 -> fc2") is the same GEMM with a relu^2
// epilogue; the down projection applies the top-k weight of each row in its
// epilogue ("Common Pitfalls" 4: routed weights on the right rows).
//
// The gate/up GEMM normally runs on two-block units (grouped_gemm_wide.cu);
// the one-block form here serves launches beyond that kernel's block limit.
//
// Tiles are token-major (block_m = 128): MMA M = 128 token rows, N = 256
// weight rows (SwiGLU: 128 gate rows followed by the matching 128 up rows, so
// one thread holds both halves of its h columns).  The down GEMM's epilogue
// is the scatter-reduce: each row's top-k-weighted output is added into an
// fp32 [T, d] accumulator at its token's row (red.global.add.v4.f32), so the
// per-slot outputs never travel through HBM; the gate/up GEMM zeroes that
// accumulator on the side (a warp of its own) and a small
// kernel converts it to bf16 afterwards.
//
// Warp roles (one CTA per SM, persistent over a static tile stride):
//   warp 0       TMA producer: weight tiles (and h tiles for the down GEMM)
//   warp 1       TMEM allocator and MMA issuer (one thread)
//   warps 2..5   epilogue: TMEM -> registers -> activation -> bf16 -> global
//                (down GEMM: warps 2..9, two per TMEM lane quadrant, each on
//                half of the tile's 256 columns)
//   warps 6..9   gate/up GEMM only: row gather of x through sorted_token_ids
//                with 16-byte cp.async into the 128B-swizzled layout (padding
//                rows zero-filled); each thread's copies of a stage arrive on
//                the stage's full barrier by cp.async.mbarrier.arrive.noinc
//   warp 10      gate/up GEMM only: zeroes the down GEMM's accumulator
// Shared-memory stages are guarded by full/empty mbarriers (TMA operands
// complete transaction bytes on the full barrier, gathered rows arrive on it
// when their copies land; the MMA thread fences the generic and async
// proxies before reading a stage), the two TMEM accumulator buffers by
// tmem-full/tmem-empty mbarriers.  Every wait is
// bounded in time; on expiry the kernel records MOE_ERR_DEVICE_TIMEOUT and
// all roles leave their loops so the CTA frees its TMEM and exits.
#include <atomic>
#include <cmath>

#include "common.cuh"
#include "gemm.h"
#include "ptx.cuh"

namespace moe {

template <int EPI>
struct GemmCfg {
  static constexpr int TOK = 128;  // token rows per tile
  // two 128-row boxes of K-major weights per stage: the gate rows and the
  // matching up rows of the tile's 128 h columns
  static constexpr bool kGated = (EPI == kEpiSwiGLU || EPI == kEpiPreSwiGLU);
  static constexpr bool kGather = (EPI == kEpiSwiGLU || EPI == kEpiRelu2);
  static constexpr bool kPre = (EPI == kEpiPreSwiGLU || EPI == kEpiPreRelu2);
  static constexpr bool kGrad = (EPI == kEpiGradSwiGLU || EPI == kEpiGradRelu2);
  static constexpr bool kReduce = (EPI == kEpiScale || EPI == kEpiDx);
  // the weight operand read MN-major: its 256 output columns are contiguous
  // in memory (W2 for dh = W2^T dout, W13 for dx = W13^T da), loaded as four
  // 64-column boxes of 64 K rows
  static constexpr bool kBmn = kGrad || EPI == kEpiDx;
  // a spare warp zeroes the accumulator the next kernel reduces into
  static constexpr bool kZero = kGather || kPre;
  static constexpr int kBoxRows = kGated ? 128 : 256;
  static constexpr int kBoxes = kGated ? 2 : 1;
  static constexpr int kWRows = kBoxRows * kBoxes;
  static constexpr int kOutCols = kBoxRows;
  static constexpr int kWBytes = kWRows * 128;
  static constexpr int kXBytes = TOK * 128;
  static constexpr int kStageBytes = kWBytes + kXBytes;
  static constexpr int kStagesRaw = (225 * 1024) / kStageBytes;
  static constexpr int kStages = kStagesRaw > 12 ? 12 : kStagesRaw;
  static constexpr int kAccCols = 256;
  static constexpr int kTmemCols = 512;
  // epilogue warps: the reductions into the fp32 accumulator, and the
  // backward's per-row fp32 reads and writes, bound those kernels, so they
  // run two warps per TMEM lane quadrant, each on half of the tile's columns
  static constexpr int kEpiWarps = (kReduce || kGrad || kPre) ? 8 : 4;
  // gate/up: warps 6-9 gather token rows, warp 10 zeroes the accumulator;
  // pre-activations: warp 6 zeroes
  static constexpr int kZeroWarp = kGather ? 10 : 2 + kEpiWarps;
  static constexpr int kNumThreads = kGather ? 352 : 64 + 32 * kEpiWarps + (kZero ? 32 : 0);
  static constexpr uint32_t kTxBytes = kWBytes + (kGather ? 0 : kXBytes);
  static constexpr int kBarrierBytes = 512;
  // reductions: per epilogue warp a 32 x 33 fp32 transpose buffer, so the
  // reduction is issued as full 128-byte row segments
  static constexpr int kRedStride = 33;
  static constexpr int kRedBytes = kReduce ? kEpiWarps * 32 * kRedStride * 4 : 0;
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024 + kBarrierBytes + kRedBytes;
  static constexpr uint32_t kIdesc = ptx::idesc_bf16_f32(128, 256, false, kBmn);

  static_assert(kStages >= 3, "pipeline depth");
  static_assert(kAccCols * 2 <= kTmemCols, "two accumulator buffers must fit TMEM");
  static_assert((2 * kStages + 5) * 8 + 16 <= kBarrierBytes, "barrier area");
  static_assert(kSmemBytes <= 232448, "shared memory per block");
};

struct TileCoord {
  int blk, wt;
  bool shared_blk;
};

// Tiles are walked in column passes of pass_w output-column tiles: all
// blocks for the first pass_w column tiles, then all blocks for the next
// ones.  Within a pass, tiles are block-major, so CTAs working together
// share an expert's weights in L2; the down GEMM picks pass_w so that one
// pass's slice of the [T, d] accumulator stays resident in L2 while it is
// being reduced into (a single pass when the whole accumulator fits).
__device__ __forceinline__ TileCoord tile_coord(int tile, int n_wt, int pass_w, int total_blocks,
                                                int routed_blocks) {
  const int per_pass = total_blocks * pass_w;
  const int pass = tile / per_pass;
  const int w0 = pass * pass_w;
  const int width = n_wt - w0 < pass_w ? n_wt - w0 : pass_w;
  const int r = tile - pass * per_pass;
  TileCoord c;
  c.blk = r / width;
  c.wt = w0 + (r - c.blk * width);
  c.shared_blk = c.blk >= routed_blocks;
  return c;
}

// silu(g) = g * sigmoid(g), with the fast approximate divide: h is rounded
// to bf16 right after, far coarser than the divide's error.
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// Named barrier 4 over the producer warp and the four gather warps, at exit.
__device__ __forceinline__ void exit_handshake() {
  __syncwarp();
  asm volatile("bar.sync 4, 160;" ::: "memory");
}

__device__ __forceinline__ void red_add_v4_f32(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

template <int EPI>
__global__ void __launch_bounds__(GemmCfg<EPI>::kNumThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ GemmArgs args) {
  using C = GemmCfg<EPI>;
  constexpr int TOK = C::TOK;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;       // the MMA issuer's last commit (drain before TMEM is freed)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* never = reinterpret_cast<volatile int*>(tmem_holder + 2);  // stays 0: drains ignore the abort
  volatile int* prod_issued = reinterpret_cast<volatile int*>(tmem_holder + 3);  // stages the producer filled

  const int warp = threadIdx.x / kWarp;
  const int lane = threadIdx.x % kWarp;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      ptx::mbar_init(&full[s], C::kGather ? 1 + 128 : 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&tfull[b], 1 + args.tfull_surplus);
      ptx::mbar_init(&tempty[b], C::kEpiWarps);
    }
    ptx::mbar_init(mma_done, 1);
    *abort_flag = 0;
    *never = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_holder, C::kTmemCols);
    ptx::tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    ptx::prefetch_tmap(&args.tm_w);
    if (args.n_shared_blocks) ptx::prefetch_tmap(&args.tm_ws);
    ptx::prefetch_tmap(&args.tm_x);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  // everything above overlaps the previous kernel; global reads start here
  pdl_wait();
  pdl_launch_dependents();
  // the router GEMM has no routed blocks: its token blocks are the
  // "shared" blocks (rows blk * 128 + r of x, the single weight matrix)
  int ntpp = EPI == kEpiRouter ? 0 : *args.ntpp;
  int routed_blocks = ntpp / args.block_m;
  if (routed_blocks < 0) routed_blocks = 0;
  if (routed_blocks > args.max_routed_blocks) routed_blocks = args.max_routed_blocks;
  const int total_blocks = routed_blocks + args.n_shared_blocks;
  const int n_wt = (args.n_out + C::kOutCols - 1) / C::kOutCols;
  const int pass_w = args.pass_cols > 0 && args.pass_cols < n_wt ? args.pass_cols : n_wt;
  const int total_tiles = total_blocks * n_wt;
  const int nk = args.K / 64;

  auto fail = [&]() {
    *abort_flag = 1;
    set_status(args.status, MOE_ERR_DEVICE_TIMEOUT);
  };

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int issued = 0;  // stages filled so far
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        const TileCoord tc = tile_coord(tile, n_wt, pass_w, total_blocks, routed_blocks);
        const CUtensorMap* tm = tc.shared_blk ? &args.tm_ws : &args.tm_w;
        int e = 0;
        if (!tc.shared_blk) {
          e = args.expert_ids[tc.blk];
          if (e < 0 || e >= args.E) set_status(args.status, MOE_ERR_BAD_EXPERT_ID);
        }
        const int row0 = tc.wt * C::kBoxRows;
        for (int kb = 0; kb < nk; ++kb) {
          if (!ptx::mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, args.wait_ns)) {
            fail();
            ok = false;
            break;
          }
          uint8_t* sW = smem + stage * C::kStageBytes;
          ptx::mbar_arrive_expect_tx(&full[stage], C::kTxBytes);
          if (C::kBmn) {
            // 64 K rows of the tile's 256 contiguous output columns, as four
            // 64-column boxes 8 KB apart (the MN-major operand's chunks)
#pragma unroll
            for (int j = 0; j < 4; ++j) ptx::tma_load_3d(sW + j * 8192, tm, &full[stage], row0 + 64 * j, kb * 64, e);
          } else {
            ptx::tma_load_3d(sW, tm, &full[stage], kb * 64, row0, e);
          }
          if (C::kGated)
            ptx::tma_load_3d(sW + C::kBoxRows * 128, tm, &full[stage], kb * 64, args.up_row_offset + row0, e);
          if (!C::kGather) ptx::tma_load_2d(sW + C::kWBytes, &args.tm_x, &full[stage], kb * 64, tc.blk * args.block_m);
          ++issued;
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      *prod_issued = issued;
    }
    // The last load into every stage lands before the CTA's shared memory is
    // released.  After an abort some were never consumed; with gathered
    // rows a stage's phase completes only with the gather warps' arrivals
    // too, so they first add the ones they did not make (exit_handshake).
    // Then the producer waits for the last phase of every stage it filled
    // (at once after a normal run, where the MMA has waited for all of them).
    if (C::kGather) {
      exit_handshake();
      exit_handshake();
    }
    if (lane == 0) {
      const int issued = *prod_issued;
      const int stage = issued % C::kStages;
      const uint32_t phase = static_cast<uint32_t>((issued / C::kStages) & 1);
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
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        if (!ptx::mbar_wait_bounded(&tempty[abuf], aphase ^ 1u, abort_flag, args.wait_ns)) {
          fail();
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(abuf * C::kAccCols);
        for (int kb = 0; kb < nk; ++kb) {
          if (!ptx::mbar_wait_bounded(&full[stage], phase, abort_flag, args.wait_ns)) {
            fail();
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          if (C::kGather) ptx::fence_proxy_async_smem();
          const uint32_t sW = ptx::smem_u32(smem + stage * C::kStageBytes);
          const uint32_t sX = sW + C::kWBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
            // B: K-major (16 K values = 32 B along the swizzled row) or
            // MN-major (16 K rows = two 1024-byte atoms)
            const uint64_t bdesc =
                C::kBmn ? ptx::sw128_mnmajor_desc(sW + kk * 2048, 8192) : ptx::sw128_kmajor_desc(sW + kk * 32);
            ptx::mma_bf16(d_tmem, ptx::sw128_kmajor_desc(sX + kk * 32), bdesc, C::kIdesc, acc);
          }
          ptx::mma_commit(&empty[stage]);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        ptx::mma_commit(&tfull[abuf]);
        if (++abuf == 2) {
          abuf = 0;
          aphase ^= 1u;
        }
      }
      // no MMA of this CTA may still run when TMEM is freed
      ptx::mma_commit(mma_done);
      if (!ptx::mbar_wait_bounded(mma_done, 0u, never, kDrainLimitNs)) fail();
    }
  } else if (warp < 2 + C::kEpiWarps) {
    // ------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const int row = q * 32 + lane;
    // with eight epilogue warps, the half of the tile's columns this warp takes
    const int ehalf = C::kEpiWarps == 8 ? (warp - 2) >> 2 : 0;
    int abuf = 0;
    uint32_t aphase = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      const TileCoord tc = tile_coord(tile, n_wt, pass_w, total_blocks, routed_blocks);
      if (!ptx::mbar_wait_bounded(&tfull[abuf], aphase, abort_flag, args.wait_ns)) {
        fail();
        break;
      }
      ptx::tc_fence_after();
      const uint32_t t_acc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(abuf * C::kAccCols);
      const int pos0 = tc.blk * args.block_m;
      // thread = token row `row` of the tile, registers = output columns
      const int p = pos0 + row;
      if (EPI == kEpiSwiGLU) {
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
          const int col = tc.wt * 128 + c0;
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
      } else if (EPI == kEpiRelu2) {
        uint16_t* orow = static_cast<uint16_t*>(args.out) + static_cast<size_t>(p) * args.n_out;
#pragma unroll 1
        for (int c0 = 0; c0 < 256; c0 += 16) {
          uint32_t a[16];
          ptx::tmem_ld16(t_acc + c0, a);
          ptx::tmem_wait_ld();
          const int col = tc.wt * 256 + c0;
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
      } else if (EPI == kEpiPreSwiGLU) {
        // pre-activations kept for the backward (fp32: the activation's
        // derivative is taken from them): g at column c, u at F + c
        float* orow = static_cast<float*>(args.out) + static_cast<size_t>(p) * args.out_ld;
#pragma unroll 1
        for (int c0 = ehalf * 64; c0 < ehalf * 64 + 64; c0 += 32) {
          uint32_t g[32], u[32];
          ptx::tmem_ld16(t_acc + c0, *reinterpret_cast<uint32_t(*)[16]>(&g[0]));
          ptx::tmem_ld16(t_acc + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&g[16]));
          ptx::tmem_ld16(t_acc + 128 + c0, *reinterpret_cast<uint32_t(*)[16]>(&u[0]));
          ptx::tmem_ld16(t_acc + 128 + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&u[16]));
          ptx::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) asm volatile("" : "+r"(g[j]), "+r"(u[j]));  // uses stay after the wait
          const int col = tc.wt * 128 + c0;
          if (col < args.n_out) {
            uint4* dg = reinterpret_cast<uint4*>(orow + col);
            uint4* du = reinterpret_cast<uint4*>(orow + args.up_row_offset + col);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              dg[i] = make_uint4(g[4 * i], g[4 * i + 1], g[4 * i + 2], g[4 * i + 3]);
              du[i] = make_uint4(u[4 * i], u[4 * i + 1], u[4 * i + 2], u[4 * i + 3]);
            }
          }
        }
      } else if (EPI == kEpiPreRelu2) {
        float* orow = static_cast<float*>(args.out) + static_cast<size_t>(p) * args.out_ld;
#pragma unroll 1
        for (int c0 = ehalf * 128; c0 < ehalf * 128 + 128; c0 += 16) {
          uint32_t a[16];
          ptx::tmem_ld16(t_acc + c0, a);
          ptx::tmem_wait_ld();
          const int col = tc.wt * 256 + c0;
          if (col < args.n_out) {
            uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(a[4 * i], a[4 * i + 1], a[4 * i + 2], a[4 * i + 3]);
          }
        }
      } else if (C::kGrad) {
        // thread = row p; TMEM columns = dhu = W2^T dout[token] for the
        // tile's 256 h columns.  With the row's top-k weight w (0 for
        // padding rows, 1 for the shared expert): dh = w * dhu, the
        // activation's derivative at the stored fp32 pre-activations gives
        // da (bf16, the operand of the dx and dW13 GEMMs), w * h goes to hw
        // (the dW2 operand), and sum(h * dhu) over the columns is this
        // tile's share of dL/dw for the row's slot.
        int slot = -1;
        float wrow = 0.0f;
        if (!tc.shared_blk) {
          slot = args.sorted_ids[p];
          if (static_cast<unsigned>(slot) < static_cast<unsigned>(args.S))
            wrow = args.topk_w[slot];
          else
            slot = -1;
        } else {
          const int t = (tc.blk - routed_blocks) * args.block_m + row;
          wrow = t < args.T ? 1.0f : 0.0f;
        }
        const float* prow = args.pre + static_cast<size_t>(p) * args.out_ld;
        uint16_t* arow = static_cast<uint16_t*>(args.out) + static_cast<size_t>(p) * args.out_ld;
        uint16_t* hrow = args.hw + static_cast<size_t>(p) * args.n_out;
        float part = 0.0f;
#pragma unroll 1
        for (int c0 = ehalf * 128; c0 < ehalf * 128 + 128; c0 += 32) {
          uint32_t a[32];
          ptx::tmem_ld16(t_acc + c0, *reinterpret_cast<uint32_t(*)[16]>(&a[0]));
          ptx::tmem_ld16(t_acc + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&a[16]));
          ptx::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) asm volatile("" : "+r"(a[j]));  // uses stay after the wait
          const int col = tc.wt * 256 + c0;
          if (col >= args.n_out) break;  // uniform across the warp
          float4 pv[8], uv[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) pv[i] = reinterpret_cast<const float4*>(prow + col)[i];
          if (EPI == kEpiGradSwiGLU) {
#pragma unroll
            for (int i = 0; i < 8; ++i) uv[i] = reinterpret_cast<const float4*>(prow + args.up_row_offset + col)[i];
          }
          const float* pg = reinterpret_cast<const float*>(pv);
          const float* pu = reinterpret_cast<const float*>(uv);
          uint32_t da_lo[16], da_hi[16], hv[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float d0[2], d1[2], hh[2];
#pragma unroll
            for (int m = 0; m < 2; ++m) {
              const int j = 2 * i + m;
              const float dhu = __uint_as_float(a[j]);
              const float dh = wrow * dhu;
              float h;
              if (EPI == kEpiGradSwiGLU) {
                const float g = pg[j];
                const float u = pu[j];
                const float sg = __frcp_rn(1.0f + __expf(-g));
                const float sl = g * sg;
                h = sl * u;
                d0[m] = dh * u * sg * (1.0f + g * (1.0f - sg));  // d/dg
                d1[m] = dh * sl;                                   // d/du
              } else {
                const float r = fmaxf(pg[j], 0.0f);
                h = r * r;
                d0[m] = 2.0f * dh * r;
                d1[m] = 0.0f;
              }
              hh[m] = wrow * h;
              part += h * dhu;
            }
            da_lo[i] = pack_bf16x2(d0[0], d0[1]);
            da_hi[i] = pack_bf16x2(d1[0], d1[1]);
            hv[i] = pack_bf16x2(hh[0], hh[1]);
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            reinterpret_cast<uint4*>(arow + col)[i] =
                make_uint4(da_lo[4 * i], da_lo[4 * i + 1], da_lo[4 * i + 2], da_lo[4 * i + 3]);
            reinterpret_cast<uint4*>(hrow + col)[i] = make_uint4(hv[4 * i], hv[4 * i + 1], hv[4 * i + 2], hv[4 * i + 3]);
            if (EPI == kEpiGradSwiGLU)
              reinterpret_cast<uint4*>(arow + args.up_row_offset + col)[i] =
                  make_uint4(da_hi[4 * i], da_hi[4 * i + 1], da_hi[4 * i + 2], da_hi[4 * i + 3]);
          }
        }
        if (slot >= 0 && args.dtopk != nullptr) atomicAdd(args.dtopk + slot, part);
      } else if (EPI == kEpiRouter) {
        // thread = token row of the tile, TMEM columns 0..E-1 = its logits,
        // written out in 16-column chunks (the routing kernel gates them:
        // a warp per token beats one thread per token working through E
        // columns in this epilogue)
        const int t = (tc.blk - routed_blocks) * args.block_m + row;
        const bool valid = t < args.T;
        const int E = args.E;
        float* lrow = args.logits + static_cast<size_t>(valid ? t : 0) * E;
#pragma unroll 1
        for (int c0 = 0; c0 < E; c0 += 16) {
          uint32_t a[16];
          ptx::tmem_ld16(t_acc + c0, a);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) asm volatile("" : "+r"(a[jj]));  // uses stay after the wait
          if (!valid) continue;
          if (c0 + 16 <= E && (E & 3) == 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              *reinterpret_cast<float4*>(lrow + c0 + 4 * i) =
                  make_float4(__uint_as_float(a[4 * i]), __uint_as_float(a[4 * i + 1]), __uint_as_float(a[4 * i + 2]),
                              __uint_as_float(a[4 * i + 3]));
          } else {
#pragma unroll
            for (int jj = 0; jj < 16; ++jj)
              if (c0 + jj < E) lrow[c0 + jj] = __uint_as_float(a[jj]);
          }
        }
      } else {
        // scatter-reduce: acc[token] += topk_weight * row (shared expert and
        // dx rows, whose da already carries the weight: 1)
        bool valid;
        int tok;
        float wrow = 1.0f;
        if (!tc.shared_blk) {
          const int slot = args.sorted_ids[p];
          valid = static_cast<unsigned>(slot) < static_cast<unsigned>(args.S);
          tok = valid ? slot / args.k : 0;
          if (valid && EPI == kEpiScale) wrow = args.topk_w[slot];
        } else {
          tok = (tc.blk - routed_blocks) * args.block_m + row;
          valid = tok < args.T;
        }
        // 32 columns at a time: each lane parks its row's 32 values in the
        // warp's transpose buffer, then 8 lanes cover one row's 128 bytes and
        // one red.v4 instruction adds 4 whole row segments
        float* stg = reinterpret_cast<float*>(smem + C::kStages * C::kStageBytes + C::kBarrierBytes) +
                     (warp - 2) * 32 * C::kRedStride;
        const int rr = lane >> 3;        // row within a group of 4
        const int cc = (lane & 7) * 4;   // column within the 32-column chunk
        // columns of this warp: all 256, or its half when two warps share a quadrant
        const int c_lo = C::kEpiWarps == 8 ? ((warp - 2) >> 2) * 128 : 0;
#pragma unroll 1
        for (int c0 = c_lo; c0 < c_lo + 256 * 4 / C::kEpiWarps; c0 += 32) {
          uint32_t a[32];
          ptx::tmem_ld16(t_acc + c0, *reinterpret_cast<uint32_t(*)[16]>(&a[0]));
          ptx::tmem_ld16(t_acc + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&a[16]));
          ptx::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) asm volatile("" : "+r"(a[j]));  // uses stay after the wait
          const int col = tc.wt * 256 + c0;
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
      if (lane == 0) ptx::mbar_arrive(&tempty[abuf]);
      if (++abuf == 2) {
        abuf = 0;
        aphase ^= 1u;
      }
    }
  } else if (C::kZero && warp == C::kZeroWarp) {
    // ------------------------------------------------ zero this CTA's share of the accumulator(s) the
    // next kernels add into (the down GEMM's, or the backward's dx and dL/dw)
    auto zero_share = [&](float* buf, int64_t n) {
      if (buf == nullptr) return;
      const int64_t per = ((n + gridDim.x - 1) / gridDim.x + 3) & ~int64_t(3);
      const int64_t lo = static_cast<int64_t>(blockIdx.x) * per;
      const int64_t hi = lo + per < n ? lo + per : n;
      for (int64_t i = lo + 4 * lane; i < hi; i += 4 * kWarp) {
        if (i + 4 <= hi)
          *reinterpret_cast<float4*>(buf + i) = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        else
          for (int64_t m = i; m < hi; ++m) buf[m] = 0.0f;
      }
    };
    zero_share(args.acc, args.acc_elems);
    zero_share(args.zero2, args.zero2_elems);
  } else if (C::kGather) {
    // ------------------------------------------------ row gather of x
    constexpr int kRowsPerThread = TOK / 16;
    const int gtid = threadIdx.x - 192;
    const int chunk = gtid & 7;
    const int r0 = gtid >> 3;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int arrived = 0;  // stages this thread has arrived on
    for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
      const TileCoord tc = tile_coord(tile, n_wt, pass_w, total_blocks, routed_blocks);
      const uint16_t* src[kRowsPerThread];
      uint32_t nbytes[kRowsPerThread];
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        const int r = r0 + 16 * i;
        int tok = 0;
        bool valid;
        if (!tc.shared_blk) {
          const int slot = args.sorted_ids[tc.blk * args.block_m + r];
          valid = static_cast<unsigned>(slot) < static_cast<unsigned>(args.S);
          if (valid) tok = slot / args.k;
        } else {
          tok = (tc.blk - routed_blocks) * args.block_m + r;
          valid = tok < args.T;
          if (!valid) tok = 0;
        }
        src[i] = args.x + static_cast<size_t>(tok) * args.K + chunk * 8;
        nbytes[i] = valid ? 16u : 0u;
      }
      for (int kb = 0; kb < nk; ++kb) {
        if (!ptx::mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, args.wait_ns)) {
          fail();
          ok = false;
          break;
        }
        const uint32_t sX = ptx::smem_u32(smem + stage * C::kStageBytes + C::kWBytes);
#pragma unroll
        for (int i = 0; i < kRowsPerThread; ++i) {
          const int r = r0 + 16 * i;
          const uint32_t dst = sX + (r >> 3) * 1024 + (r & 7) * 128 + ((chunk ^ (r & 7)) << 4);
          ptx::cp_async_16(dst, src[i] + kb * 64, nbytes[i]);
        }
        ptx::cp_async_arrive_noinc(&full[stage]);
        ++arrived;
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // this thread's rows have landed
    // after an abort: arrive on every stage the producer filled and this
    // thread did not, so that the producer can wait for its own loads
    exit_handshake();
    for (const int target = *prod_issued; arrived < target; ++arrived) {
      ptx::mbar_arrive(&full[stage]);
      if (++stage == C::kStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    exit_handshake();
  }

  // every warp reconverges (the idle lanes of the producer and MMA warps
  // wait for their working lane) before the block-wide barrier
  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ---------------------------------------------------------------- host side

namespace {

template <int EPI>
cudaError_t launch_variant(const GemmArgs& args, int grid, cudaStream_t stream) {
  using C = GemmCfg<EPI>;
  auto kern = grouped_gemm_kernel<EPI>;
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

int gemm_box_rows(int epi) { return (epi == kEpiSwiGLU || epi == kEpiPreSwiGLU) ? 128 : 256; }

int64_t gemm_max_tiles(int epi, int max_routed_blocks, int n_shared_blocks, int n_out) {
  const int cols = gemm_box_rows(epi);
  const int64_t n_wt = (n_out + cols - 1) / cols;
  return static_cast<int64_t>(max_routed_blocks + n_shared_blocks) * n_wt;
}

cudaError_t launch_grouped_gemm(int epi, const GemmArgs& a, int grid, cudaStream_t s) {
  if (a.block_m != 128) return cudaErrorInvalidValue;
  switch (epi) {
    case kEpiSwiGLU: return launch_variant<kEpiSwiGLU>(a, grid, s);
    case kEpiRelu2: return launch_variant<kEpiRelu2>(a, grid, s);
    case kEpiScale: return launch_variant<kEpiScale>(a, grid, s);
    case kEpiRouter: return launch_variant<kEpiRouter>(a, grid, s);
    case kEpiPreSwiGLU: return launch_variant<kEpiPreSwiGLU>(a, grid, s);
    case kEpiPreRelu2: return launch_variant<kEpiPreRelu2>(a, grid, s);
    case kEpiGradSwiGLU: return launch_variant<kEpiGradSwiGLU>(a, grid, s);
    case kEpiGradRelu2: return launch_variant<kEpiGradRelu2>(a, grid, s);
    case kEpiDx: return launch_variant<kEpiDx>(a, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace moe
