// Gate/up (or fc1) grouped GEMM on 256-token tiles: the "Grouped GEMM
// Structure" of the fused-moe-kernel page ("Fused MoE Kernel Optimization",
// skillmd zjli2013) with the activation of the axolotl `_moe_triton_forward`
// (act_fn(gate) * up) or the squared ReLU of the mlxcel PR in the epilogue,
// for token rows gathered straight from x.
//
// A tile is a "unit" of one or two consecutive 128-row blocks of the same
// expert (a unit starts at the first block of an expert's run and at every
// second block after it; the shared expert's blocks are one run) times 256
// weight rows.  Each K step stages the 256 weight rows once (TMA) and the
// unit's token rows (cp.async gather, up to 256), and the MMA thread issues
// two M = 128, N = 256 MMAs that share the weight operand: per SM a 64-wide
// K step writes 64 KB into shared memory (and the MMAs read 96 KB) for two
// 128 x 256 products, against 48 KB (and 48 KB) for one in the one-block
// kernel.  Shared-memory traffic, staging writes plus operand reads, is what
// bounds these single-CTA GEMMs.
// The two accumulators fill all 512 TMEM columns, so the accumulator is not
// double-buffered: at the end of a tile the eight epilogue warps drain block
// 0's accumulator, then block 1's; the MMA thread starts the next tile's
// block 0 as soon as the first is drained and lets it run up to two K steps
// ahead of block 1 (those stages stay held) until the second is.
//
// Warp roles (one CTA per SM, persistent over a static tile stride):
//   warp 0        TMA producer: weight tiles (gate rows and matching up rows)
//   warp 1        TMEM allocator and MMA issuer (one thread)
//   warps 2..5    epilogue (one TMEM lane quadrant each; first half of the columns)
//   warps 6..9    row gather of x through sorted_token_ids (16-byte cp.async
//                 into the 128B-swizzled layout; padding rows zero-filled),
//                 arriving on the stage's full barrier when the copies land
//   warp 10       zeroes the down GEMM's fp32 accumulator on the side
//   warps 11..14  epilogue (second half of the columns)
// Every pipeline wait is bounded in time; on expiry the kernel records
// MOE_ERR_DEVICE_TIMEOUT, drains its own loads and MMAs, frees its tensor
// memory and returns.
#include <atomic>

#include "common.cuh"
#include "gemm.h"
#include "ptx.cuh"

namespace moe {

template <int EPI>
struct WideCfg {
  static constexpr bool kGated = EPI == kEpiSwiGLU;
  static constexpr int kBoxRows = kGated ? 128 : 256;  // weight rows per TMA box
  static constexpr int kOutCols = kBoxRows;            // h columns per tile
  static constexpr int kWBytes = 256 * 128;            // 256 weight rows x 64 K (bf16)
  static constexpr int kXBytes = 128 * 128;            // one block's 128 token rows x 64 K
  static constexpr int kStageBytes = kWBytes + 2 * kXBytes;
  static constexpr int kStages = 3;
  static constexpr int kBarrierBytes = 256;
  static constexpr int kUnitBytes = kWideMaxBlocks * 2;  // first block of each unit (uint16)
  static constexpr int kSmemBytes = kStages * kStageBytes + kBarrierBytes + kUnitBytes + 1024;
  static constexpr int kNumThreads = 480;
  static constexpr int kTmemCols = 512;
  static constexpr uint32_t kIdesc = ptx::idesc_bf16_f32(128, 256);
  static_assert(kSmemBytes <= 232448, "shared memory per block");
  static_assert(kWideMaxBlocks * 4 <= kStages * kStageBytes, "expert-id scratch fits the stages");
  static_assert(kWideMaxBlocks <= 65536, "unit table entries are 16-bit");
};

__device__ __forceinline__ float silu_w(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// Named barrier 4 over the producer warp and the four gather warps, at exit.
__device__ __forceinline__ void wide_exit_handshake() {
  __syncwarp();
  asm volatile("bar.sync 4, 160;" ::: "memory");
}

template <int EPI>
__global__ void __launch_bounds__(WideCfg<EPI>::kNumThreads, 1)
    grouped_gemm_wide_kernel(const __grid_constant__ GemmArgs args) {
  using C = WideCfg<EPI>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 1;       // [2]: block 0's and block 1's accumulator drained
  uint64_t* mma_done = tempty + 2;    // the MMA issuer's last commit (drain before TMEM is freed)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* never = reinterpret_cast<volatile int*>(tmem_holder + 2);  // stays 0: drains ignore the abort
  volatile int* prod_issued = reinterpret_cast<volatile int*>(tmem_holder + 3);
  int* n_units_smem = reinterpret_cast<int*>(tmem_holder + 4);
  uint16_t* unit_b0 = reinterpret_cast<uint16_t*>(smem + C::kStages * C::kStageBytes + C::kBarrierBytes);
  int* eid = reinterpret_cast<int*>(smem);  // expert of every block, before the stages are used

  const int warp = threadIdx.x / kWarp;
  const int lane = threadIdx.x % kWarp;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      ptx::mbar_init(&full[s], 1 + 128);  // producer's expect_tx + one arrival per gather thread
      ptx::mbar_init(&empty[s], 1);
    }
    ptx::mbar_init(tfull, 1 + args.tfull_surplus);
    ptx::mbar_init(&tempty[0], 8);  // the eight epilogue warps
    ptx::mbar_init(&tempty[1], 8);
    ptx::mbar_init(mma_done, 1);
    *abort_flag = 0;
    *never = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&args.tm_w);
    if (args.n_shared_blocks) ptx::prefetch_tmap(&args.tm_ws);
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_holder, C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  // everything above overlaps the previous kernel; global reads start here
  pdl_wait();
  pdl_launch_dependents();
  int routed_blocks = *args.ntpp / args.block_m;
  if (routed_blocks < 0) routed_blocks = 0;
  if (routed_blocks > args.max_routed_blocks) routed_blocks = args.max_routed_blocks;
  const int total_blocks = routed_blocks + args.n_shared_blocks;  // <= kWideMaxBlocks (host check)

  // ---- units: every thread loads a share of the block experts, then one
  // warp marks unit starts (first block of a run of equal experts, and every
  // second block after it) and compacts them in order
  for (int b = threadIdx.x; b < total_blocks; b += C::kNumThreads)
    eid[b] = b < routed_blocks ? args.expert_ids[b] : INT32_MIN;  // the shared expert's run
  __syncthreads();
  if (warp == 0) {
    int run_start = 0, n_units = 0, prev_e = 0;
    for (int base = 0; base < total_blocks; base += kWarp) {
      const int b = base + lane;
      const bool in = b < total_blocks;
      const int e = in ? eid[b] : 0;
      const int up = __shfl_up_sync(0xffffffffu, e, 1);
      const int left = lane == 0 ? prev_e : up;
      const bool head = in && (b == 0 || b == routed_blocks || e != left);
      const unsigned heads = __ballot_sync(0xffffffffu, head);
      const unsigned upto = heads & (0xffffffffu >> (31 - lane));
      const int my_run = upto ? base + (31 - __clz(upto)) : run_start;
      const bool start = in && ((b - my_run) & 1) == 0;
      const unsigned starts = __ballot_sync(0xffffffffu, start);
      if (start) unit_b0[n_units + __popc(starts & ((1u << lane) - 1u))] = static_cast<uint16_t>(b);
      n_units += __popc(starts);
      run_start = __shfl_sync(0xffffffffu, my_run, 31);
      prev_e = __shfl_sync(0xffffffffu, e, 31);
    }
    if (lane == 0) *n_units_smem = n_units;
  }
  __syncthreads();
  const int n_units = *n_units_smem;
  const int n_wt = (args.n_out + C::kOutCols - 1) / C::kOutCols;
  const int total_tiles = n_units * n_wt;
  const int nk = args.K / 64;

  // tile -> (first block, blocks in the unit, weight tile); unit-major, so
  // the CTAs working together share the unit's gathered rows and the
  // expert's weights in L2
  struct Tile {
    int b0, nb, wt;
    bool shared_blk;
  };
  auto tile_of = [&](int tile) {
    Tile t;
    const int u = tile / n_wt;
    t.wt = tile - u * n_wt;
    t.b0 = unit_b0[u];
    const int next = u + 1 < n_units ? static_cast<int>(unit_b0[u + 1]) : total_blocks;
    t.nb = next - t.b0 >= 2 ? 2 : 1;
    t.shared_blk = t.b0 >= routed_blocks;
    return t;
  };
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
      int issued = 0;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        const Tile t = tile_of(tile);
        const CUtensorMap* tm = t.shared_blk ? &args.tm_ws : &args.tm_w;
        int e = 0;
        if (!t.shared_blk) {
          e = args.expert_ids[t.b0];
          if (e < 0 || e >= args.E) set_status(args.status, MOE_ERR_BAD_EXPERT_ID);
        }
        const int row0 = t.wt * C::kBoxRows;
        for (int kb = 0; kb < nk; ++kb) {
          if (!ptx::mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, args.wait_ns)) {
            fail();
            ok = false;
            break;
          }
          uint8_t* sW = smem + stage * C::kStageBytes;
          ptx::mbar_arrive_expect_tx(&full[stage], C::kWBytes);
          ptx::tma_load_3d(sW, tm, &full[stage], kb * 64, row0, e);
          if (C::kGated)
            ptx::tma_load_3d(sW + C::kBoxRows * 128, tm, &full[stage], kb * 64, args.up_row_offset + row0, e);
          ++issued;
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      *prod_issued = issued;
    }
    // The last load into every stage lands before the shared memory is
    // released; after an abort the gather warps first add the arrivals they
    // did not make on the stages the producer filled (see the gather role).
    wide_exit_handshake();
    wide_exit_handshake();
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
      uint32_t tph = 0;  // parity of the accumulator's current use
      bool ok = true;
      // the four MMAs of one 64-wide K step of block `blk` (its accumulator
      // at TMEM column blk * 256), from stage `st`
      auto mma_block = [&](int st, int kb, int blk) {
        const uint32_t sW = ptx::smem_u32(smem + st * C::kStageBytes);
        const uint32_t sX = sW + C::kWBytes + blk * C::kXBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::mma_bf16(tmem_base + static_cast<uint32_t>(blk * 256), ptx::sw128_kmajor_desc(sX + kk * 32),
                        ptx::sw128_kmajor_desc(sW + kk * 32), C::kIdesc, (kb | kk) != 0 ? 1u : 0u);
      };
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        const Tile t = tile_of(tile);
        // block 0's accumulator is free once the epilogue has drained it
        if (!ptx::mbar_wait_bounded(&tempty[0], tph ^ 1u, abort_flag, args.wait_ns)) {
          fail();
          break;
        }
        ptx::tc_fence_after();
        // While the epilogue still drains block 1's accumulator, block 0
        // runs ahead: up to kStages - 1 leading K steps keep their stage
        // until block 1's MMAs for them are issued.
        bool d1_free = false;
        int deferred = 0;
        const int s_first = stage;
        auto flush = [&]() {
          ptx::tc_fence_after();
          d1_free = true;
          for (int j = 0; j < deferred; ++j) {
            const int sj = (s_first + j) % C::kStages;
            mma_block(sj, j, 1);
            ptx::mma_commit(&empty[sj]);
          }
          deferred = 0;
        };
        for (int kb = 0; kb < nk; ++kb) {
          if (!ptx::mbar_wait_bounded(&full[stage], phase, abort_flag, args.wait_ns)) {
            fail();
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          ptx::fence_proxy_async_smem();  // gathered rows were written by the generic proxy
          mma_block(stage, kb, 0);
          bool release = true;
          if (t.nb == 2) {
            if (!d1_free) {
              if (ptx::mbar_try_wait(&tempty[1], tph ^ 1u)) {
                flush();
              } else if (deferred < C::kStages - 1) {
                ++deferred;
                release = false;
              } else if (ptx::mbar_wait_bounded(&tempty[1], tph ^ 1u, abort_flag, args.wait_ns)) {
                flush();
              } else {
                fail();
                ok = false;
                break;
              }
            }
            if (d1_free) mma_block(stage, kb, 1);
          }
          if (release) ptx::mma_commit(&empty[stage]);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        // every tile takes one phase of both accumulators' barriers
        if (!d1_free) {
          if (!ptx::mbar_wait_bounded(&tempty[1], tph ^ 1u, abort_flag, args.wait_ns)) {
            fail();
            break;
          }
          flush();
        }
        ptx::mma_commit(tfull);
        tph ^= 1u;
      }
      // no MMA of this CTA may still run when TMEM is freed
      ptx::mma_commit(mma_done);
      if (!ptx::mbar_wait_bounded(mma_done, 0u, never, kDrainLimitNs)) fail();
    }
  } else if ((warp >= 2 && warp < 6) || warp >= 11) {
    // ------------------------------------------------ epilogue: block 0's rows, then block 1's
    const int half = warp >= 11 ? 1 : 0;  // two warps per TMEM lane quadrant, each on half the columns
    const int q = warp & 3;               // TMEM lane quadrant this warp may access
    const int row = q * 32 + lane;
    uint32_t tph = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      const Tile t = tile_of(tile);
      if (!ptx::mbar_wait_bounded(tfull, tph, abort_flag, args.wait_ns)) {
        fail();
        break;
      }
      ptx::tc_fence_after();
      for (int blk = 0; blk < 2; ++blk) {
        if (blk < t.nb) {
          const uint32_t t_acc =
              tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(blk * 256);
          const int p = (t.b0 + blk) * args.block_m + row;
          uint16_t* orow = static_cast<uint16_t*>(args.out) + static_cast<size_t>(p) * args.n_out;
          if (EPI == kEpiSwiGLU) {
            // 32 h columns per TMEM wait (F is a multiple of 64, so a chunk
            // is either wholly inside the layer or wholly past it)
#pragma unroll 1
            for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32) {
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
                  const float h0 = silu_w(__uint_as_float(g[2 * i])) * __uint_as_float(u[2 * i]);
                  const float h1 = silu_w(__uint_as_float(g[2 * i + 1])) * __uint_as_float(u[2 * i + 1]);
                  pk[i] = pack_bf16x2(h0, h1);
                }
                uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                  dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
              }
            }
          } else {
#pragma unroll 1
            for (int c0 = half * 128; c0 < half * 128 + 128; c0 += 32) {
              uint32_t a[32];
              ptx::tmem_ld16(t_acc + c0, *reinterpret_cast<uint32_t(*)[16]>(&a[0]));
              ptx::tmem_ld16(t_acc + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&a[16]));
              ptx::tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 32; ++j) asm volatile("" : "+r"(a[j]));  // uses stay after the wait
              const int col = t.wt * 256 + c0;
              if (col < args.n_out) {
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                  const float v0 = fmaxf(__uint_as_float(a[2 * i]), 0.0f);
                  const float v1 = fmaxf(__uint_as_float(a[2 * i + 1]), 0.0f);
                  pk[i] = pack_bf16x2(v0 * v0, v1 * v1);
                }
                uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                  dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
              }
            }
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&tempty[blk]);
      }
      tph ^= 1u;
    }
  } else if (warp == 10) {
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
  } else {
    // ------------------------------------------------ row gather of x (warps 6..9)
    // thread: one 16-byte chunk (of the row's 128-byte K step) of 16 rows
    constexpr int kRows = 16;
    const int gtid = threadIdx.x - 6 * kWarp;
    const int chunk = gtid & 7;
    const int r0 = gtid >> 3;  // rows r0, r0 + 16, ..., r0 + 240 of the unit
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int arrived = 0;
    for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
      const Tile t = tile_of(tile);
      const uint16_t* src[kRows];
      uint32_t nbytes[kRows];
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        const int r = r0 + 16 * i;
        const int blk = t.b0 + (r >> 7);
        int tok = 0;
        bool valid = (r >> 7) < t.nb;
        if (valid) {
          if (!t.shared_blk) {
            const int slot = args.sorted_ids[blk * args.block_m + (r & 127)];
            valid = static_cast<unsigned>(slot) < static_cast<unsigned>(args.S);
            if (valid) tok = slot / args.k;
          } else {
            tok = (blk - routed_blocks) * args.block_m + (r & 127);
            valid = tok < args.T;
            if (!valid) tok = 0;
          }
        }
        src[i] = args.x + static_cast<size_t>(tok) * args.K + chunk * 8;
        nbytes[i] = valid ? 16u : 0u;
      }
      const int rows_live = t.nb * 128;
      for (int kb = 0; kb < nk; ++kb) {
        if (!ptx::mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, args.wait_ns)) {
          fail();
          ok = false;
          break;
        }
        const uint32_t sX = ptx::smem_u32(smem + stage * C::kStageBytes + C::kWBytes);
#pragma unroll
        for (int i = 0; i < kRows; ++i) {
          const int r = r0 + 16 * i;
          if (r < rows_live) {
            const uint32_t dst = sX + (r >> 3) * 1024 + (r & 7) * 128 + ((chunk ^ (r & 7)) << 4);
            ptx::cp_async_16(dst, src[i] + kb * 64, nbytes[i]);
          }
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
    wide_exit_handshake();
    for (const int target = *prod_issued; arrived < target; ++arrived) {
      ptx::mbar_arrive(&full[stage]);
      if (++stage == C::kStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    wide_exit_handshake();
  }

  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

namespace {

template <int EPI>
cudaError_t launch_wide_variant(const GemmArgs& args, int grid, cudaStream_t stream) {
  using C = WideCfg<EPI>;
  auto kern = grouped_gemm_wide_kernel<EPI>;
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

bool gemm_wide_supported(int epi, int block_m, int total_blocks_max) {
  return (epi == kEpiSwiGLU || epi == kEpiRelu2) && block_m == 128 && total_blocks_max <= kWideMaxBlocks;
}

cudaError_t launch_grouped_gemm_wide(int epi, const GemmArgs& a, int grid, cudaStream_t s) {
  if (!gemm_wide_supported(epi, a.block_m, a.max_routed_blocks + a.n_shared_blocks)) return cudaErrorInvalidValue;
  if (epi == kEpiSwiGLU) return launch_wide_variant<kEpiSwiGLU>(a, grid, s);
  return launch_wide_variant<kEpiRelu2>(a, grid, s);
}

}  // namespace moe
