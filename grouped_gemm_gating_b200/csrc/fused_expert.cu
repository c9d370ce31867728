// Fused expert kernel for small token blocks (block_m = 16..64): the gate/up
// GEMM with its activation, the down GEMM with the top-k weights and, for
// small batches, the scatter-reduce, in one persistent launch.
//
// This is the same computation as the separate grouped GEMMs (see
// grouped_gemm.cu for the sources: "Grouped GEMM Structure" of the
// fused-moe-kernel page, the gate/up, activation, down and weighted-sum
// sequence of the axolotl `_moe_triton_forward`, the relu^2 experts of the
// mlxcel PR) specialised for the decode / verifier shape, where the layer is
// bound by streaming each hit expert's weights once from HBM and every
// separate launch costs as much as a few microseconds of that stream.
//
// Work list: all gate/up tiles (block, h-column tile) first, then all down
// tiles (block, d-column tile).  Every CTA walks the list with the same
// static stride, so its own gate/up tiles always come before its down tiles
// and no CTA waits on work queued behind itself; all CTAs are co-resident
// (one per SM, grid <= SM count).  A down tile needs the block's full h rows:
// the gate/up epilogue publishes each finished tile (h stores, a barrier of
// the epilogue warps, then one red.release.gpu add on ready[block]); every
// token-loader thread polls ready[block] with ld.acquire.gpu and then loads
// its share of the block's h rows with cp.async.  No GPU-scope fence sits on this path: such fences wait
// behind the SM's queue of in-flight weight loads.  The weight warp streams
// the down tile's W2 slices without waiting, so the down GEMM's weight
// traffic overlaps the tail of the gate/up phase.  Every stage is signalled
// as soon as its bytes land (TMA transaction bytes for weights,
// cp.async.mbarrier.arrive.noinc for token rows), so no warp holds back a
// stage that another tile needs while it waits.
//
// Combine (do_combine, T*k <= 64, no shared expert): the CTA that finishes
// the last down tile of a d-column tile (done[column tile] reaches the
// number of blocks) sums, for that column range, out[t] = sum_j
// y[inv_pos[t*k + j]] in fp32 in slot order and writes bf16 -- the same
// arithmetic as the combine kernel; all its loads are issued before the
// first sum so the tail costs two memory round trips.
//
// Every wait is bounded in time; on expiry the kernel records
// MOE_ERR_DEVICE_TIMEOUT and all roles leave their loops.
#include "common.cuh"
#include "fused.h"
#include "gemm.h"
#include "ptx.cuh"

namespace moe {

namespace {

template <int EPI1, int TOK>
struct FusedCfg {
  static constexpr bool kGated = (EPI1 == kEpiSwiGLU);
  // Every stage holds 128 weight rows: SwiGLU gate/up tiles stack 64 gate
  // rows on the 64 matching up rows (one M = 128 MMA, 64 h columns per
  // tile); relu^2 fc1 tiles and down tiles hold 128 rows of one matrix.
  static constexpr int kWRows = 128;
  static constexpr int kH1Cols = kGated ? 64 : 128;  // h columns per gate/up tile
  static constexpr int kWBytes = kWRows * 128;
  static constexpr int kXBytes = TOK * 128;
  static constexpr int kStageBytes = kWBytes + kXBytes;
  static constexpr int kXbufBytes = kGated ? 64 * TOK * 4 : 0;  // up half handed to the gate half
  static constexpr int kStagesRaw = (225 * 1024 - kXbufBytes) / kStageBytes;
  static constexpr int kStages = kStagesRaw > 12 ? 12 : kStagesRaw;
  static constexpr int kAccCols = TOK;
  static constexpr int kTmemNeed = 2 * kAccCols;
  static constexpr int kTmemCols = kTmemNeed <= 32    ? 32
                                   : kTmemNeed <= 64  ? 64
                                   : kTmemNeed <= 128 ? 128
                                   : kTmemNeed <= 256 ? 256
                                                      : 512;
  static constexpr int kNumThreads = 320;
  static constexpr uint32_t kTx = kWBytes;
  static constexpr int kBarrierBytes = 256;
  static constexpr int kSlotBytes = 256;  // inv_pos of the in-kernel combine (64 slots)
  static constexpr int kSmemBytes = kStages * kStageBytes + kXbufBytes + kSlotBytes + 1024 + kBarrierBytes;
  static constexpr uint32_t kIdesc = ptx::idesc_bf16_f32(128, TOK);
  static_assert(TOK == 16 || TOK == 32 || TOK == 64, "token rows per tile");
  static_assert(kStageBytes % 1024 == 0, "stages stay 1024-byte aligned");
  static_assert(kStages >= 3, "pipeline depth");
  static_assert((2 * kStages + 4) * 8 + 16 <= kBarrierBytes, "barrier area");  // + 4 words
  static_assert(kSmemBytes <= 232448, "shared memory per block");
};

struct Tile {
  int phase;  // 1: gate/up, 2: down
  int blk, wt;
  bool shared_blk;
};

__device__ __forceinline__ Tile fused_tile(int u, int n1_tiles, int n_wt1, int n_wt2, int routed_blocks) {
  Tile t;
  if (u < n1_tiles) {
    t.phase = 1;
    t.blk = u / n_wt1;
    t.wt = u - t.blk * n_wt1;
  } else {
    const int v = u - n1_tiles;
    t.phase = 2;
    t.blk = v / n_wt2;
    t.wt = v - t.blk * n_wt2;
  }
  t.shared_blk = t.blk >= routed_blocks;
  return t;
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

// Slots (T * k) up to which the kernel does the scatter-reduce itself.
constexpr int kCombineMaxSlots = 64;

// Named barrier 1 over the four epilogue warps (barrier 0 is
// __syncthreads).  Each warp reconverges first, as the aligned barrier
// requires.  epilogue_any() is the same barrier with an OR reduction: the
// epilogue takes its leave-on-timeout decision uniformly, so no epilogue
// thread can be left waiting at a later barrier for one that left.
__device__ __forceinline__ void epilogue_sync() {
  __syncwarp();
  asm volatile("bar.sync 1, 128;" ::: "memory");
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

template <int EPI1, int TOK>
__global__ void __launch_bounds__(FusedCfg<EPI1, TOK>::kNumThreads, 1)
    fused_expert_kernel(const __grid_constant__ FusedArgs args) {
  using C = FusedCfg<EPI1, TOK>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* xbuf = reinterpret_cast<float*>(smem + C::kStages * C::kStageBytes);  // [TOK][64]
  int* s_slot = reinterpret_cast<int*>(smem + C::kStages * C::kStageBytes + C::kXbufBytes);
  uint64_t* full =
      reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes + C::kXbufBytes + C::kSlotBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_holder + 2);

  const int warp = threadIdx.x / kWarp;
  const int lane = threadIdx.x % kWarp;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      ptx::mbar_init(&full[s], 1 + 128);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&tfull[b], 1);
      ptx::mbar_init(&tempty[b], 4);
    }
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&args.tm_w13);
    ptx::prefetch_tmap(&args.tm_w2);
    if (args.n_shared_blocks) {
      ptx::prefetch_tmap(&args.tm_w13s);
      ptx::prefetch_tmap(&args.tm_w2s);
    }
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_holder, C::kTmemCols);
    ptx::tmem_relinquish();
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
  const int total_blocks = routed_blocks + args.n_shared_blocks;
  const int n_wt1 = (args.F + C::kH1Cols - 1) / C::kH1Cols;
  const int n_wt2 = (args.d + 127) / 128;
  const int n1_tiles = total_blocks * n_wt1;
  const int total_tiles = n1_tiles + total_blocks * n_wt2;
  const int nk1 = args.d / 64;
  const int nk2 = args.F / 64;

  auto fail = [&]() {
    *abort_flag = 1;
    set_status(args.status, MOE_ERR_DEVICE_TIMEOUT);
  };

  if (warp == 0) {
    // ------------------------------------------------ TMA producer (weights)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < total_tiles; u += gridDim.x) {
        const Tile t = fused_tile(u, n1_tiles, n_wt1, n_wt2, routed_blocks);
        int e = 0;
        if (!t.shared_blk) {
          e = args.expert_ids[t.blk];
          if (e < 0 || e >= args.E) set_status(args.status, MOE_ERR_BAD_EXPERT_ID);
        }
        const int nk = t.phase == 1 ? nk1 : nk2;
        const CUtensorMap* tm = t.phase == 1 ? (t.shared_blk ? &args.tm_w13s : &args.tm_w13)
                                             : (t.shared_blk ? &args.tm_w2s : &args.tm_w2);
        for (int kb = 0; kb < nk; ++kb) {
          if (!ptx::mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, kWaitLimitNs)) {
            fail();
            ok = false;
            break;
          }
          uint8_t* sW = smem + stage * C::kStageBytes;
          ptx::mbar_arrive_expect_tx(&full[stage], C::kTx);
          if (t.phase == 1 && C::kGated) {
            // 64 gate rows, then the 64 matching up rows (64-row boxes)
            ptx::tma_load_3d(sW, tm, &full[stage], kb * 64, t.wt * 64, e);
            ptx::tma_load_3d(sW + 64 * 128, tm, &full[stage], kb * 64, args.F + t.wt * 64, e);
          } else {
            ptx::tma_load_3d(sW, tm, &full[stage], kb * 64, t.wt * 128, e);
          }
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
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
      for (int u = blockIdx.x; ok && u < total_tiles; u += gridDim.x) {
        const Tile t = fused_tile(u, n1_tiles, n_wt1, n_wt2, routed_blocks);
        if (!ptx::mbar_wait_bounded(&tempty[abuf], aphase ^ 1u, abort_flag, kWaitLimitNs)) {
          fail();
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(abuf * C::kAccCols);
        const int nk = t.phase == 1 ? nk1 : nk2;
        for (int kb = 0; kb < nk; ++kb) {
          if (!ptx::mbar_wait_bounded(&full[stage], phase, abort_flag, kWaitLimitNs)) {
            fail();
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          ptx::fence_proxy_async_smem();
          const uint32_t sW = ptx::smem_u32(smem + stage * C::kStageBytes);
          const uint32_t sX = sW + C::kWBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
            const uint64_t dw = ptx::sw128_kmajor_desc(sW + kk * 32);
            const uint64_t dx = ptx::sw128_kmajor_desc(sX + kk * 32);
            ptx::mma_bf16(d_tmem, dw, dx, C::kIdesc, acc);
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
    }
  } else if (warp < 6) {
    // ------------------------------------------------ epilogue
    const int q = warp & 3;
    const int row = q * 32 + lane;  // weight row within the tile = output column
    const int etid = threadIdx.x - 64;
    int abuf = 0;
    uint32_t aphase = 0;
    for (int u = blockIdx.x; u < total_tiles; u += gridDim.x) {
      const Tile t = fused_tile(u, n1_tiles, n_wt1, n_wt2, routed_blocks);
      const bool got = ptx::mbar_wait_bounded(&tfull[abuf], aphase, abort_flag, kWaitLimitNs);
      if (epilogue_any(!got)) {
        if (!got) fail();
        break;
      }
      ptx::tc_fence_after();
      const uint32_t t_acc =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(abuf * C::kAccCols);
      const int pos0 = t.blk * args.block_m;
      if (t.phase == 1 && C::kGated) {
        // lanes 0-63 hold the gate and lanes 64-127 the up pre-activations
        // of h columns wt*64 + (row % 64): the up half goes through xbuf
        const int col = t.wt * 64 + (row & 63);
        const bool col_ok = col < args.F;
        float gate[TOK];
#pragma unroll
        for (int j0 = 0; j0 < TOK; j0 += 16) {
          uint32_t a[16];
          ptx::tmem_ld16(t_acc + j0, a);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            if (q >= 2)
              xbuf[(j0 + jj) * 64 + (row - 64)] = __uint_as_float(a[jj]);
            else
              gate[j0 + jj] = __uint_as_float(a[jj]);
          }
        }
        epilogue_sync();
        if (q < 2 && col_ok) {
#pragma unroll
          for (int j = 0; j < TOK; ++j)
            args.h[static_cast<size_t>(pos0 + j) * args.F + col] =
                float_to_bf16_bits(silu_f(gate[j]) * xbuf[j * 64 + row]);
        }
      } else if (t.phase == 1) {
        const int col = t.wt * 128 + row;
        const bool col_ok = col < args.F;
#pragma unroll 1
        for (int j0 = 0; j0 < TOK; j0 += 16) {
          uint32_t a[16];
          ptx::tmem_ld16(t_acc + j0, a);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            float v = fmaxf(__uint_as_float(a[jj]), 0.0f);
            v *= v;
            if (col_ok) args.h[static_cast<size_t>(pos0 + j0 + jj) * args.F + col] = float_to_bf16_bits(v);
          }
        }
      } else {
        const int col = t.wt * 128 + row;
        const bool col_ok = col < args.d;
#pragma unroll 1
        for (int j0 = 0; j0 < TOK; j0 += 16) {
          uint32_t a[16];
          ptx::tmem_ld16(t_acc + j0, a);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const int p = pos0 + j0 + jj;
            bool valid;
            float wv = 1.0f;
            if (!t.shared_blk) {
              const int slot = args.sorted_ids[p];
              valid = static_cast<unsigned>(slot) < static_cast<unsigned>(args.S);
              if (valid) wv = args.topk_w[slot];
            } else {
              valid = (t.blk - routed_blocks) * args.block_m + j0 + jj < args.T;
            }
            if (col_ok && valid) args.y[static_cast<size_t>(p) * args.d + col] = __uint_as_float(a[jj]) * wv;
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&tempty[abuf]);
      if (++abuf == 2) {
        abuf = 0;
        aphase ^= 1u;
      }
      // publish the finished tile: the barrier orders every epilogue
      // thread's stores before thread 0's GPU-scope release
      epilogue_sync();
      if (t.phase == 1) {
        if (etid == 0) ptx::red_release_gpu_add(&args.ready[t.blk], 1);
      } else if (args.do_combine) {
        if (etid == 0) *last_flag = (ptx::atom_acq_rel_gpu_add(&args.done[t.wt], 1) == total_blocks - 1) ? 1 : 0;
        epilogue_sync();
        if (*last_flag) {
          // this CTA finished the last down tile of column tile t.wt (its
          // acquire plus the barrier order the loads below after every
          // other CTA's y stores): every load first, then the sums in order
          const int c = t.wt * 128 + row;
          const int nslot = args.T * args.k;
          for (int i = etid; i < nslot; i += 128) s_slot[i] = __ldcg(args.inv_pos + i);
          epilogue_sync();
          if (c < args.d) {
            float v[kCombineMaxSlots];
#pragma unroll
            for (int i = 0; i < kCombineMaxSlots; ++i)
              if (i < nslot) v[i] = __ldcg(args.y + static_cast<size_t>(s_slot[i]) * args.d + c);
            float acc = 0.0f;
            int j = 0, tok = 0;
#pragma unroll
            for (int i = 0; i < kCombineMaxSlots; ++i) {
              if (i < nslot) {
                acc += v[i];
                if (++j == args.k) {
                  args.out[static_cast<size_t>(tok) * args.d + c] = float_to_bf16_bits(acc);
                  acc = 0.0f;
                  j = 0;
                  ++tok;
                }
              }
            }
          }
        }
      }
    }
  } else {
    // ------------------------------------------------ token operand
    // 128 threads copy the tile's token rows with cp.async: gathered x rows
    // for gate/up tiles, the block's h rows for down tiles once published
    constexpr int kRowsPerThread = TOK / 16;
    const int gtid = threadIdx.x - 192;
    const int chunk = gtid & 7;
    const int r0 = gtid >> 3;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < total_tiles; u += gridDim.x) {
      const Tile t = fused_tile(u, n1_tiles, n_wt1, n_wt2, routed_blocks);
      const uint16_t* src[kRowsPerThread];
      uint32_t nbytes[kRowsPerThread];
      int K;
      if (t.phase == 1) {
        K = args.d;
#pragma unroll
        for (int i = 0; i < kRowsPerThread; ++i) {
          const int r = r0 + 16 * i;
          int tok = 0;
          bool valid;
          if (!t.shared_blk) {
            const int slot = args.sorted_ids[t.blk * args.block_m + r];
            valid = static_cast<unsigned>(slot) < static_cast<unsigned>(args.S);
            if (valid) tok = slot / args.k;
          } else {
            tok = (t.blk - routed_blocks) * args.block_m + r;
            valid = tok < args.T;
            if (!valid) tok = 0;
          }
          src[i] = args.x + static_cast<size_t>(tok) * K + chunk * 8;
          nbytes[i] = valid ? 16u : 0u;
        }
      } else {
        K = args.F;
        // wait until every gate/up tile of this block has published its h
        // (this thread holds no unsignalled stage while it waits)
        const uint64_t t0 = ptx::globaltimer_ns();
        while (ptx::ld_acquire_gpu(args.ready + t.blk) < n_wt1) {
          if (*abort_flag || ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
            fail();
            ok = false;
            break;
          }
          __nanosleep(128);
        }
        if (!ok) break;
#pragma unroll
        for (int i = 0; i < kRowsPerThread; ++i) {
          const int r = r0 + 16 * i;
          src[i] = args.h + static_cast<size_t>(t.blk * args.block_m + r) * K + chunk * 8;
          nbytes[i] = 16u;
        }
      }
      const int nk = K / 64;
      for (int kb = 0; kb < nk; ++kb) {
        if (!ptx::mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, kWaitLimitNs)) {
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
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
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
  // Check out; the last CTA returns every counter to zero for the next
  // launch (no other CTA touches them any more).
  if (threadIdx.x == 0)
    *last_flag = ptx::atom_acq_rel_gpu_add(args.finished, 1) == static_cast<int>(gridDim.x) - 1 ? 1 : 0;
  __syncthreads();
  if (*last_flag) {
    for (int i = threadIdx.x; i < total_blocks; i += blockDim.x) args.ready[i] = 0;
    for (int i = threadIdx.x; i < n_wt2; i += blockDim.x) args.done[i] = 0;
    if (threadIdx.x == 0) *args.finished = 0;
  }
}

template <int EPI1, int TOK>
cudaError_t launch_fused_variant(const FusedArgs& args, int grid, cudaStream_t stream) {
  using C = FusedCfg<EPI1, TOK>;
  auto kern = fused_expert_kernel<EPI1, TOK>;
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_done[dev]) {
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (err != cudaSuccess) return err;
    attr_done[dev] = true;
  }
  return launch_pdl(kern, dim3(grid), dim3(C::kNumThreads), C::kSmemBytes, stream, args);
}

}  // namespace

bool fused_expert_supported(int block_m) { return block_m == 16 || block_m == 32 || block_m == 64; }

bool fused_expert_combines(int T, int k, int n_shared) {
  return n_shared == 0 && static_cast<int64_t>(T) * k <= kCombineMaxSlots;
}

cudaError_t launch_fused_expert(int act_epi, int block_m, const FusedArgs& args, int grid, cudaStream_t stream) {
  const bool gated = act_epi == kEpiSwiGLU;
  switch (block_m) {
    case 16: return gated ? launch_fused_variant<kEpiSwiGLU, 16>(args, grid, stream)
                          : launch_fused_variant<kEpiRelu2, 16>(args, grid, stream);
    case 32: return gated ? launch_fused_variant<kEpiSwiGLU, 32>(args, grid, stream)
                          : launch_fused_variant<kEpiRelu2, 32>(args, grid, stream);
    case 64: return gated ? launch_fused_variant<kEpiSwiGLU, 64>(args, grid, stream)
                          : launch_fused_variant<kEpiRelu2, 64>(args, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace moe
