// gemm_sm100.cuh — bf16 GEMM C = A · Wᵀ with fp32 accumulation on the sm_100a tensor cores.
//
// The HSTU layer around the attention (DLRMv3 review, section "model selection", FLOP-formula
// paragraph: per layer 2·(L²·D/2 + 4·L·D² + 3·L·D²) flops) spends its non-attention work in dense
// projections of the L token rows.  This kernel computes one such projection: A is [M, K] (token
// rows), W is [N, K] (the weight in the out-features × in-features layout of a linear layer), C is
// [M, N]; all bf16, row-major.
//
// Persistent and warp-specialised, one CTA per SM:
//   warp 0       TMA producer: 128×64 tiles of A and 256×64 tiles of W into a 4-stage ring
//                (128-byte swizzle, K-major, zero fill past the edges);
//   warp 1       MMA issuer: per 64-deep k block four tcgen05.mma 128×256×16 (each instruction
//                carries 128 clocks of tensor work, so the issuing thread has slack for its
//                waits and commits) into one of two TMEM accumulators of 256 columns;
//   warps 2..5   epilogue: TMEM -> registers -> bf16 -> row- and column-predicated 32-byte stores
//                (16-byte ones when N is not a multiple of 16 or C is not 32-byte aligned),
//                overlapping the next tile's main loop on the other accumulator.
// Output tiles are visited in N-fastest order: CTAs working at the same time share one A tile (the
// large operand: token rows), while W, a few MB for a layer's projection, stays in L2 throughout.
// Every wait is bounded; a timeout sets the error word and the kernel drains and returns.
#pragma once

#include "hstu_fwd_sm100.cuh"

namespace hstu {

constexpr int kGemmBM = 128;
constexpr int kGemmBN = 256;
constexpr int kGemmBK = 64;  // one 128-byte swizzle atom of bf16
constexpr int kGemmStages = 4;
constexpr int kGemmThreads = 192;

struct GemmCfg {
  static constexpr int kABytes = kGemmBM * kGemmBK * 2;  // 16 KB
  static constexpr int kBBytes = kGemmBN * kGemmBK * 2;  // 32 KB
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kSmemBytes = 1024 + kGemmStages * kStageBytes + 1024;
  static constexpr uint32_t kIdesc = ptx::idesc_bf16_f32(kGemmBM, kGemmBN, false);
};

struct GemmCtl {
  uint64_t full[kGemmStages], empty[kGemmStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int32_t abort_flag;
};

struct GemmParams {
  __nv_bfloat16* c;
  int32_t M, N, K;
  int32_t tiles_m, tiles_n;
  unsigned* err;
};

// 32 bytes to global memory in one instruction (st.global.v8.b32); the address is 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void* p, const uint4& a, const uint4& b) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a.x), "r"(a.y),
               "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
               : "memory");
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w,
                     const GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  const uint32_t sbase = ptx::smem_addr(smem);
  auto* ctl = reinterpret_cast<GemmCtl*>(smem + kGemmStages * GemmCfg::kStageBytes);
  volatile int32_t* abort_flag = &ctl->abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  auto bar = [](const uint64_t& b) { return ptx::smem_addr(&b); };
  auto sA = [&](int s) { return sbase + s * GemmCfg::kStageBytes; };
  auto sB = [&](int s) { return sbase + s * GemmCfg::kStageBytes + GemmCfg::kABytes; };

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      ptx::mbar_init(bar(ctl->full[s]), 1);
      ptx::mbar_init(bar(ctl->empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(bar(ctl->acc_full[a]), 1);
      ptx::mbar_init(bar(ctl->acc_empty[a]), 4);  // one arrival per epilogue warp
    }
    ptx::mbar_init(bar(ctl->drain), 1);
    ctl->abort_flag = 0;
    ptx::fence_mbarrier_init();
    ptx::prefetch_tmap(&tm_a);
    ptx::prefetch_tmap(&tm_w);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_addr(&ctl->tmem_base), 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  // Launched as a programmatic dependent: A may come from the previous kernel, and C may be memory
  // it still reads, so nothing global is touched before that kernel has completed.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  const int ntiles = p.tiles_m * p.tiles_n;
  const int kblocks = (p.K + kGemmBK - 1) / kGemmBK;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const int m0 = (tile / p.tiles_n) * kGemmBM;
        const int n0 = (tile % p.tiles_n) * kGemmBN;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!wait_bounded(bar(ctl->empty[stage]), phase ^ 1u, abort_flag, p.err)) {
            ok = false;
            break;
          }
          const uint32_t fb = bar(ctl->full[stage]);
          ptx::mbar_arrive_expect_tx(fb, GemmCfg::kStageBytes);
          ptx::tma_load_2d(sA(stage), &tm_a, fb, kb * kGemmBK, m0);
          ptx::tma_load_2d(sB(stage), &tm_w, fb, kb * kGemmBK, n0);
          ++issued;
          if (++stage == kGemmStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (*abort_flag) {
        // Let every copy this CTA started land before its shared memory is released.
        for (int k = 1; k <= kGemmStages && k <= issued; ++k) {
          const int pos = issued - k;
          drain_wait(bar(ctl->full[pos % kGemmStages]), (uint32_t)((pos / kGemmStages) & 1));
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    const uint32_t lead = (lane == 0) ? 1u : 0u;
    auto wait_all = [&](uint32_t b, uint32_t par) {
      return __all_sync(0xffffffffu, wait_bounded(b, par, abort_flag, p.err));
    };
    int stage = 0;
    uint32_t phase = 0;
    uint32_t acc_empty_par[2] = {1u, 1u};
    int acc = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
      ok = wait_all(bar(ctl->acc_empty[acc]), acc_empty_par[acc]);
      if (!ok) break;
      acc_empty_par[acc] ^= 1u;
      ptx::tc_fence_after();
      const uint32_t dacc = tmem + acc * kGemmBN;
      for (int kb = 0; kb < kblocks; ++kb) {
        ok = wait_all(bar(ctl->full[stage]), phase);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint64_t da = ptx::smem_desc(sA(stage), 16, 1024, 2);
        const uint64_t db = ptx::smem_desc(sB(stage), 16, 1024, 2);
#pragma unroll
        for (int ks = 0; ks < kGemmBK / 16; ++ks)  // +32 bytes along the swizzled row per k step
          ptx::mma_ss_lead(lead, dacc, da + ks * 2, db + ks * 2, GemmCfg::kIdesc, (kb | ks) ? 1u : 0u);
        ptx::mma_commit_lead(lead, bar(ctl->empty[stage]));
        if (++stage == kGemmStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      ptx::mma_commit_lead(lead, bar(ctl->acc_full[acc]));
      acc ^= 1;
    }
    ptx::mma_commit_lead(lead, bar(ctl->drain));
    drain_wait(bar(ctl->drain), 0u);
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..5)
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    uint32_t acc_full_par[2] = {0u, 0u};
    int acc = 0;
    // 32-byte stores fill whole sectors; they need N % 16 == 0 and a 32-byte aligned C.
    const bool wide_stores = (p.N % 16 == 0) && ((reinterpret_cast<uintptr_t>(p.c) & 31u) == 0);
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
      ok = __all_sync(0xffffffffu, wait_bounded(bar(ctl->acc_full[acc]), acc_full_par[acc], abort_flag, p.err));
      if (!ok) break;
      acc_full_par[acc] ^= 1u;
      ptx::tc_fence_after();
      const int m = (tile / p.tiles_n) * kGemmBM + row;
      const int n0 = (tile % p.tiles_n) * kGemmBN;
      __nv_bfloat16* dst = p.c + (size_t)(m < p.M ? m : 0) * p.N + n0;
#pragma unroll 1
      for (int c = 0; c < kGemmBN / 32; ++c) {
        uint32_t r[32];
        ptx::tmem_ld32(tmem + lane_off + acc * kGemmBN + c * 32, r);
        ptx::tmem_ld_wait(r);
        if (m < p.M) {
          uint4 v[4];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            v[q4].x = pack_bf16x2(__uint_as_float(r[q4 * 8 + 0]), __uint_as_float(r[q4 * 8 + 1]));
            v[q4].y = pack_bf16x2(__uint_as_float(r[q4 * 8 + 2]), __uint_as_float(r[q4 * 8 + 3]));
            v[q4].z = pack_bf16x2(__uint_as_float(r[q4 * 8 + 4]), __uint_as_float(r[q4 * 8 + 5]));
            v[q4].w = pack_bf16x2(__uint_as_float(r[q4 * 8 + 6]), __uint_as_float(r[q4 * 8 + 7]));
          }
          if (wide_stores) {
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2)
              if (n0 + c * 32 + h2 * 16 < p.N) st_global_v8(dst + c * 32 + h2 * 16, v[2 * h2], v[2 * h2 + 1]);
          } else {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              if (n0 + c * 32 + q4 * 8 < p.N) *reinterpret_cast<uint4*>(dst + c * 32 + q4 * 8) = v[q4];
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(ctl->acc_empty[acc]));
      acc ^= 1;
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, 512);
}


// ---------------------------------------------------------------------------------------------
// Two-SM form: C tiles of 256 × 256 computed by a cluster of two CTAs on paired SMs.
//
// CTA r of the pair loads rows [128 r, 128 r + 128) of the tile's A rows and of its W rows (half
// of N), 128 × 64 each per k block, into the same shared-memory offsets.  One thread of CTA 0
// issues tcgen05.mma.cta_group::2 with M = 256, N = 256: each SM multiplies its own A rows by all
// 256 W rows, reading the other half of W from the peer's shared memory, and accumulates its 128
// rows × 256 columns in its own TMEM.  Per flop this moves two thirds of the operand bytes of the
// one-SM 128 × 256 tile, from L2 and into shared memory.
//
//   warp 0      producer (both CTAs): waits until the stage is free (the MMA commit arrives on
//               `empty` of both CTAs), then TMA-loads its two halves.  Both CTAs' copies complete
//               on CTA 0's `full`, which CTA 0's producer arms with the bytes of all four;
//   warp 1      CTA 0: MMA issuer; commits to `empty` and `acc_full` of both CTAs.  (A relay in
//               which CTA 1 waited on its own barrier and then arrived on CTA 0's cost one
//               cluster-scope round trip per stage and halved the throughput.)
//   warps 2..5  epilogue (both CTAs): its 128 rows of the accumulator, then an arrival on CTA 0's
//               `acc_empty` (eight arrivals: four warps in each CTA), released at CTA scope.  Eight warps, two per TMEM
//               lane quarter, measured no faster.
// Every wait is bounded; on a timeout the CTA records it, leaves its loops and drains, and the
// peer's waits on it run out in turn.
// ---------------------------------------------------------------------------------------------
constexpr int kGemm2BM = 256;  // rows of A per cluster tile (128 per CTA)
constexpr int kGemm2BN = 256;  // rows of W per cluster tile (128 per CTA)
constexpr int kGemm2Stages = 6;
constexpr int kGemm2EpiWarps = 4;
constexpr int kGemm2Threads = 64 + 32 * kGemm2EpiWarps;

struct Gemm2Cfg {
  static constexpr int kHalfBytes = 128 * kGemmBK * 2;  // 16 KB: 128 rows × 64 of A or of W
  static constexpr int kStageBytes = 2 * kHalfBytes;    // one CTA's copies of a stage
  static constexpr int kSmemBytes = 1024 + kGemm2Stages * kStageBytes + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory");
  static constexpr uint32_t kIdesc = ptx::idesc_bf16_f32(kGemm2BM, kGemm2BN, false);
};

struct Gemm2Ctl {
  uint64_t full[kGemm2Stages], empty[kGemm2Stages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int32_t abort_flag;
};

// Bounded wait whose acquire is at cluster scope: for barriers that the peer CTA's threads arrive on.
__device__ __noinline__ bool wait_bounded_cluster_slow(uint32_t bar, uint32_t parity, volatile int32_t* abort_flag,
                                                       unsigned* err) {
  const uint64_t t0 = ptx::globaltimer_ns();
  while (true) {
    if (ptx::mbar_try_wait_cluster(bar, parity, 0xffffffffu)) return true;
    if (*abort_flag) return false;
    if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicOr(err, kErrTimeout);
      return false;
    }
  }
}
__device__ __forceinline__ bool wait_bounded_cluster(uint32_t bar, uint32_t parity, volatile int32_t* abort_flag,
                                                     unsigned* err) {
  if (ptx::mbar_try_wait_cluster(bar, parity, 0xffffffffu)) return true;
  return wait_bounded_cluster_slow(bar, parity, abort_flag, err);
}

__global__ void __launch_bounds__(kGemm2Threads, 1)
    gemm_bf16_2sm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w,
                         const GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  const uint32_t sbase = ptx::smem_addr(smem);
  auto* ctl = reinterpret_cast<Gemm2Ctl*>(smem + kGemm2Stages * Gemm2Cfg::kStageBytes);
  volatile int32_t* abort_flag = &ctl->abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  auto bar = [](const uint64_t& b) { return ptx::smem_addr(&b); };
  auto sA = [&](int s) { return sbase + s * Gemm2Cfg::kStageBytes; };
  auto sB = [&](int s) { return sbase + s * Gemm2Cfg::kStageBytes + Gemm2Cfg::kHalfBytes; };

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kGemm2Stages; ++s) {
      ptx::mbar_init(bar(ctl->full[s]), 1);
      ptx::mbar_init(bar(ctl->empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(bar(ctl->acc_full[a]), 1);
      ptx::mbar_init(bar(ctl->acc_empty[a]), 2 * kGemm2EpiWarps);  // every epilogue warp of both CTAs
    }
    ptx::mbar_init(bar(ctl->drain), 1);
    ctl->abort_flag = 0;
    ptx::fence_mbarrier_init();
    ptx::prefetch_tmap(&tm_a);
    ptx::prefetch_tmap(&tm_w);
  }
  if (warp == 1) {
    ptx::tmem_alloc_2sm(ptx::smem_addr(&ctl->tmem_base), 512);
    ptx::tmem_relinquish_2sm();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // the peer's barriers are initialised before anything arrives on them
  ptx::tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  // Launched as a programmatic dependent: A may come from the previous kernel, and C may be memory
  // it still reads, so nothing global is touched before that kernel has completed.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  const int ntiles = p.tiles_m * p.tiles_n;
  const int kblocks = (p.K + kGemmBK - 1) / kGemmBK;
  const int cluster = (int)ptx::cluster_id_x();
  const int nclusters = (int)ptx::nclusters_x();

  if (warp == 0) {
    // ------------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int tile = cluster; tile < ntiles && ok; tile += nclusters) {
        const int m0 = (tile / p.tiles_n) * kGemm2BM + 128 * (int)rank;
        const int n0 = (tile % p.tiles_n) * kGemm2BN + 128 * (int)rank;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!wait_bounded(bar(ctl->empty[stage]), phase ^ 1u, abort_flag, p.err)) {
            ok = false;
            break;
          }
          if (rank == 0) ptx::mbar_arrive_expect_tx(bar(ctl->full[stage]), 2 * Gemm2Cfg::kStageBytes);
          const uint32_t fb = ptx::mapa_shared(bar(ctl->full[stage]), 0);
          ptx::tma_load_2d_2sm(sA(stage), &tm_a, fb, kb * kGemmBK, m0);
          ptx::tma_load_2d_2sm(sB(stage), &tm_w, fb, kb * kGemmBK, n0);
          ++issued;
          if (++stage == kGemm2Stages) { stage = 0; phase ^= 1u; }
        }
      }
      if (*abort_flag) {
        if (rank == 0) {
          // Both CTAs' copies of a stage complete CTA 0's `full`: wait for the last stages armed.
          for (int k = 1; k <= kGemm2Stages && k <= issued; ++k) {
            const int pos = issued - k;
            drain_wait(bar(ctl->full[pos % kGemm2Stages]), (uint32_t)((pos / kGemm2Stages) & 1));
          }
        } else {
          // CTA 1 cannot wait on the barrier its copies complete on (it lives in CTA 0), so it
          // gives them kCopyGraceNs to land (a copy takes microseconds) before it leaves.
          const uint64_t t0 = ptx::globaltimer_ns();
          while (ptx::globaltimer_ns() - t0 < kCopyGraceNs) {
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (CTA 0 only)
    if (rank == 0) {
      const uint32_t lead = (lane == 0) ? 1u : 0u;
      auto wait_all = [&](uint32_t b, uint32_t par) {
        return __all_sync(0xffffffffu, wait_bounded(b, par, abort_flag, p.err));
      };
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_empty_par[2] = {1u, 1u};
      int acc = 0;
      bool ok = true;
      for (int tile = cluster; tile < ntiles && ok; tile += nclusters) {
        ok = __all_sync(0xffffffffu,
                        wait_bounded_cluster(bar(ctl->acc_empty[acc]), acc_empty_par[acc], abort_flag, p.err));
        if (!ok) break;
        acc_empty_par[acc] ^= 1u;
        ptx::tc_fence_after();
        const uint32_t dacc = tmem + acc * kGemm2BN;
        for (int kb = 0; kb < kblocks; ++kb) {
          ok = wait_all(bar(ctl->full[stage]), phase);
          if (!ok) break;
          ptx::tc_fence_after();
          const uint64_t da = ptx::smem_desc(sA(stage), 16, 1024, 2);
          const uint64_t db = ptx::smem_desc(sB(stage), 16, 1024, 2);
#pragma unroll
          for (int ks = 0; ks < kGemmBK / 16; ++ks)  // +32 bytes along the swizzled row per k step
            ptx::mma_ss_2sm_lead(lead, dacc, da + ks * 2, db + ks * 2, Gemm2Cfg::kIdesc, (kb | ks) ? 1u : 0u);
          ptx::mma_commit_2sm_lead(lead, bar(ctl->empty[stage]), 3);
          if (++stage == kGemm2Stages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        ptx::mma_commit_2sm_lead(lead, bar(ctl->acc_full[acc]), 3);
        acc ^= 1;
      }
      ptx::mma_commit_2sm_lead(lead, bar(ctl->drain), 1);
      drain_wait(bar(ctl->drain), 0u);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..)
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    constexpr int kCols = kGemm2BN * 4 / kGemm2EpiWarps;  // columns per warp
    const int col0 = ((warp - 2) / 4) * kCols;
    uint32_t acc_full_par[2] = {0u, 0u};
    int acc = 0;
    const bool wide_stores = (p.N % 16 == 0) && ((reinterpret_cast<uintptr_t>(p.c) & 31u) == 0);
    bool ok = true;
    for (int tile = cluster; tile < ntiles; tile += nclusters) {
      ok = __all_sync(0xffffffffu, wait_bounded(bar(ctl->acc_full[acc]), acc_full_par[acc], abort_flag, p.err));
      if (!ok) break;
      acc_full_par[acc] ^= 1u;
      ptx::tc_fence_after();
      const int m = (tile / p.tiles_n) * kGemm2BM + 128 * (int)rank + row;
      const int n0 = (tile % p.tiles_n) * kGemm2BN + col0;
      __nv_bfloat16* dst = p.c + (size_t)(m < p.M ? m : 0) * p.N + n0;
#pragma unroll 1
      for (int c = 0; c < kCols / 32; ++c) {
        uint32_t r[32];
        ptx::tmem_ld32(tmem + lane_off + acc * kGemm2BN + col0 + c * 32, r);
        ptx::tmem_ld_wait(r);
        if (m < p.M) {
          uint4 v[4];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            v[q4].x = pack_bf16x2(__uint_as_float(r[q4 * 8 + 0]), __uint_as_float(r[q4 * 8 + 1]));
            v[q4].y = pack_bf16x2(__uint_as_float(r[q4 * 8 + 2]), __uint_as_float(r[q4 * 8 + 3]));
            v[q4].z = pack_bf16x2(__uint_as_float(r[q4 * 8 + 4]), __uint_as_float(r[q4 * 8 + 5]));
            v[q4].w = pack_bf16x2(__uint_as_float(r[q4 * 8 + 6]), __uint_as_float(r[q4 * 8 + 7]));
          }
          if (wide_stores) {
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2)
              if (n0 + c * 32 + h2 * 16 < p.N) st_global_v8(dst + c * 32 + h2 * 16, v[2 * h2], v[2 * h2 + 1]);
          } else {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              if (n0 + c * 32 + q4 * 8 < p.N) *reinterpret_cast<uint4*>(dst + c * 32 + q4 * 8) = v[q4];
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      // Release at CTA scope, not cluster scope: the latter held each warp until its 64 KB of C
      // stores were visible and cost the K = 512 projection a fifth of its throughput.
      if (lane == 0) ptx::mbar_arrive_remote(ptx::mapa_shared(bar(ctl->acc_empty[acc]), 0));
      acc ^= 1;
    }
  }

  // Neither CTA leaves (nor frees TMEM) while the other may still read its shared memory or
  // arrive on its barriers.
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc_2sm(tmem, 512);
}

}  // namespace hstu
