// hstu_bwd_dq_sm100.cuh — the dQ half of the backward pass from stored dS tiles, for sm_100a.
//
// Forward (DLRMv3 review, section "model selection"): out = Mask(SiLU(alpha Q K^T)) V / N.  By the
// chain rule dQ_i = sum over visible keys j of dS_ij k_j.  The dK/dV kernel forms every dS tile
// anyway; when a workspace is given it also writes each one there (bf16, as the MMAs use it), and
// this kernel only multiplies: per query tile qt and head,
//     dQ[qt] = sum over the visible key tiles kt of dS(kt, qt) K[kt]
// with no score MMAs and no elementwise work.  The stored tile is dS^T (rows = keys, columns =
// queries), so dS enters the MMA as an MN-major A operand, and K as an MN-major B operand, both
// straight from TMA tiles.
//
//   warp 0      producer: fetches the next item (user, query tile, head) from the cost-ordered
//               list, then streams (dS tile, K tile) pairs of its visible key tiles through a ring.
//   warp 1      MMA issuer (lane 0 issues): 8 MMAs (K = 16 keys each) per pair into one of two
//               TMEM accumulators, so the epilogue of one item overlaps the next item's MMAs.
//   warps 2-5   epilogue: dQ rows from TMEM -> bf16 -> row-predicated stores.
//
// Waits are bounded as in the other kernels; on expiry the kernel reports, drains and returns.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "bwd_schedule.cuh"
#include "hstu_fwd_sm100.cuh"
#include "sm100_ptx.cuh"

namespace hstu {

template <int D>
struct DqCfg {
  using T = FwdCfg<D>;                                // K tile geometry
  static constexpr int kDsBlockBytes = kTileRows * 128;  // 128 rows x 64 bf16, 128-byte swizzle
  static constexpr int kDsBytes = 2 * kDsBlockBytes;      // a 128 x 128 bf16 dS tile
  static constexpr int kStageBytes = kDsBytes + T::kTileBytes;
  static constexpr int kStages = (D == 128) ? 3 : 4;
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory");
  static constexpr uint32_t kTmemCols = (2 * D < 32) ? 32u : static_cast<uint32_t>(2 * D);
  static constexpr uint32_t kIdesc = ptx::idesc_bf16_f32_ab(128, D, true, true);
};

constexpr int kDqThreads = 192;
constexpr int kDqSlots = 4;

struct DqParams {
  const int32_t* seq_offsets;
  const int32_t* num_targets;  // may be null
  const int4* items;           // {b, query tile, h, cost}
  const int32_t* num_items;
  int32_t* work_counter;
  int32_t* done_counter;
  const long long* ds_base;    // [B+1] first dS tile of each user (all heads)
  __nv_bfloat16* dq;
  int32_t H;
  unsigned* err;
};

template <int kStages>
struct DqCtl {
  uint64_t full[kStages], empty[kStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t sched_full[kDqSlots], sched_empty[kDqSlots];
  uint64_t drain;
  // work slot: valid, b, h, qt, row0, L, U, e1, s2, e2
  int32_t slot[kDqSlots][10];
  uint32_t tmem_base;
  int32_t abort_flag;
};

struct DqWork {
  int valid, b, h, qt, row0, L, U;
  TileRange r;
};

__device__ __forceinline__ DqWork read_dq_slot(const volatile int32_t* s) {
  DqWork w;
  w.valid = s[0];
  w.b = s[1];
  w.h = s[2];
  w.qt = s[3];
  w.row0 = s[4];
  w.L = s[5];
  w.U = s[6];
  w.r.e1 = s[7];
  w.r.s2 = s[8];
  w.r.e2 = s[9];
  return w;
}

template <int D>
__global__ void __launch_bounds__(kDqThreads, 1)
    hstu_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_ds, const __grid_constant__ CUtensorMap tm_k,
                       const DqParams p) {
  using Cfg = DqCfg<D>;
  using T = typename Cfg::T;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  const uint32_t sbase = ptx::smem_addr(smem);
  auto* ctl = reinterpret_cast<DqCtl<Cfg::kStages>*>(smem + Cfg::kStages * Cfg::kStageBytes);
  volatile int32_t* abort_flag = &ctl->abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  auto bar = [](const uint64_t& b) { return ptx::smem_addr(&b); };
  auto sDs = [&](int s) { return sbase + s * Cfg::kStageBytes; };
  auto sK = [&](int s) { return sbase + s * Cfg::kStageBytes + Cfg::kDsBytes; };

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < Cfg::kStages; ++s) {
      ptx::mbar_init(bar(ctl->full[s]), 1);
      ptx::mbar_init(bar(ctl->empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(bar(ctl->acc_full[a]), 1);
      ptx::mbar_init(bar(ctl->acc_empty[a]), 4);  // one arrival per epilogue warp
    }
    for (int s = 0; s < kDqSlots; ++s) {
      ptx::mbar_init(bar(ctl->sched_full[s]), 1);
      ptx::mbar_init(bar(ctl->sched_empty[s]), 1 + 4);  // MMA warp and epilogue warps
    }
    ptx::mbar_init(bar(ctl->drain), 1);
    ctl->abort_flag = 0;
    ptx::fence_mbarrier_init();
    ptx::prefetch_tmap(&tm_ds);
    ptx::prefetch_tmap(&tm_k);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_addr(&ctl->tmem_base), Cfg::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      asm volatile("griddepcontrol.wait;" ::: "memory");
      const int M = *p.num_items;
      int slot = 0;
      uint32_t sched_empty_par = (1u << kDqSlots) - 1u;
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      while (ok) {
        const int idx = atomicAdd(p.work_counter, 1);
        DqWork w{};
        w.valid = idx < M;
        long long base = 0;  // this user's and head's first dS tile
        if (w.valid) {
          const int4 it = p.items[idx];
          w.b = it.x;
          w.qt = it.y;
          w.h = it.z;
          w.row0 = p.seq_offsets[w.b];
          w.L = p.seq_offsets[w.b + 1] - w.row0;
          w.U = w.L - (p.num_targets ? p.num_targets[w.b] : 0);
          w.r = key_tiles_of_query_tile(w.qt, w.L, w.U);
          base = p.ds_base[w.b] + (long long)w.h * ds_tiles_per_head(w.L, w.U);
        }
        if (!wait_bounded(bar(ctl->sched_empty[slot]), (sched_empty_par >> slot) & 1u, abort_flag, p.err)) {
          ok = false;
          break;
        }
        sched_empty_par ^= 1u << slot;
        volatile int32_t* s = ctl->slot[slot];
        s[0] = w.valid; s[1] = w.b; s[2] = w.h; s[3] = w.qt; s[4] = w.row0;
        s[5] = w.L; s[6] = w.U; s[7] = w.r.e1; s[8] = w.r.s2; s[9] = w.r.e2;
        ptx::mbar_arrive(bar(ctl->sched_full[slot]));
        slot = (slot + 1) & (kDqSlots - 1);
        if (!w.valid) break;

        const int n = tile_count(w.r);
        for (int i = 0; i < n; ++i) {
          const int kt = tile_at(w.r, i);
          const long long tile = base + ds_tiles_before(kt, w.L, w.U) + (w.qt - kt);
          if (!wait_bounded(bar(ctl->empty[stage]), phase ^ 1u, abort_flag, p.err)) {
            ok = false;
            break;
          }
          const uint32_t fb = bar(ctl->full[stage]);
          ptx::mbar_arrive_expect_tx(fb, Cfg::kStageBytes);
          for (int blk = 0; blk < 2; ++blk)
            ptx::tma_load_2d(sDs(stage) + blk * Cfg::kDsBlockBytes, &tm_ds, fb, blk * 64,
                             static_cast<int32_t>(tile * kTileRows));
          for (int blk = 0; blk < T::kBlocks; ++blk)
            ptx::tma_load_2d(sK(stage) + blk * T::kBlockBytes, &tm_k, fb, w.h * D + blk * T::kBlockElems,
                             w.row0 + kt * kTileRows);
          ++issued;
          if (++stage == Cfg::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag) {
        // Let every copy this CTA started land before its shared memory is released.
        for (int k = 1; k <= Cfg::kStages && k <= issued; ++k) {
          const int pos = issued - k;
          drain_wait(bar(ctl->full[pos % Cfg::kStages]), (uint32_t)((pos / Cfg::kStages) & 1));
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
    int slot = 0;
    uint32_t sched_full_par = 0u;
    int stage = 0;
    uint32_t phase = 0;
    uint32_t acc_empty_par[2] = {1u, 1u};
    int acc = 0;
    bool ok = true;
    while (ok) {
      if (!wait_all(bar(ctl->sched_full[slot]), (sched_full_par >> slot) & 1u)) {
        ok = false;
        break;
      }
      sched_full_par ^= 1u << slot;
      const DqWork w = read_dq_slot(ctl->slot[slot]);
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(ctl->sched_empty[slot]));
      slot = (slot + 1) & (kDqSlots - 1);
      if (!w.valid) break;
      if (!wait_all(bar(ctl->acc_empty[acc]), acc_empty_par[acc])) {
        ok = false;
        break;
      }
      acc_empty_par[acc] ^= 1u;
      const uint32_t dacc = tmem + acc * D;
      const int n = tile_count(w.r);
      for (int i = 0; i < n; ++i) {
        if (!wait_all(bar(ctl->full[stage]), phase)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        // dS^T tile: queries contiguous in 64-element atoms 16 KB apart, 16 keys = 2 KB per K step.
        const uint64_t da = ptx::smem_desc(sDs(stage), Cfg::kDsBlockBytes, 1024, 2);
        // K tile: head columns contiguous, one 128-byte (or 64-byte) row per key.
        const uint64_t db = ptx::smem_desc(sK(stage), T::kBlockBytes, 8 * T::kRowBytes, T::kSwizzle);
#pragma unroll
        for (int ks = 0; ks < kTileRows / 16; ++ks)
          ptx::mma_ss_lead(lead, dacc, da + ((ks * 16 * 128) >> 4), db + ((ks * 16 * T::kRowBytes) >> 4),
                           Cfg::kIdesc, (i | ks) ? 1u : 0u);
        ptx::mma_commit_lead(lead, bar(ctl->empty[stage]));
        if (++stage == Cfg::kStages) {
          stage = 0;
          phase ^= 1u;
        }
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
    int slot = 0;
    uint32_t sched_full_par = 0u;
    uint32_t acc_full_par[2] = {0u, 0u};
    int acc = 0;
    bool ok = true;
    while (ok) {
      ok = __all_sync(0xffffffffu, wait_bounded(bar(ctl->sched_full[slot]), (sched_full_par >> slot) & 1u,
                                                abort_flag, p.err));
      if (!ok) break;
      sched_full_par ^= 1u << slot;
      const DqWork w = read_dq_slot(ctl->slot[slot]);
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(ctl->sched_empty[slot]));
      slot = (slot + 1) & (kDqSlots - 1);
      if (!w.valid) break;
      ok = __all_sync(0xffffffffu, wait_bounded(bar(ctl->acc_full[acc]), acc_full_par[acc], abort_flag, p.err));
      if (!ok) break;
      acc_full_par[acc] ^= 1u;
      ptx::tc_fence_after();
      const bool live = w.qt * kTileRows + row < w.L;
      const size_t grow = (size_t)(w.row0 + w.qt * kTileRows + row);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ro[32];
        ptx::tmem_ld32(tmem + lane_off + acc * D + 32 * c, ro);
        ptx::tmem_ld_wait(ro);
        if (live) {
          uint4* d4 = reinterpret_cast<uint4*>(p.dq + (grow * p.H + w.h) * D + 32 * c);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(ro[q4 * 8 + 0]), __uint_as_float(ro[q4 * 8 + 1]));
            v.y = pack_bf16x2(__uint_as_float(ro[q4 * 8 + 2]), __uint_as_float(ro[q4 * 8 + 3]));
            v.z = pack_bf16x2(__uint_as_float(ro[q4 * 8 + 4]), __uint_as_float(ro[q4 * 8 + 5]));
            v.w = pack_bf16x2(__uint_as_float(ro[q4 * 8 + 6]), __uint_as_float(ro[q4 * 8 + 7]));
            d4[q4] = v;
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
  if (warp == 1) ptx::tmem_dealloc(tmem, Cfg::kTmemCols);
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.done_counter, 1) == (int)gridDim.x - 1) {
      atomicExch(p.work_counter, 0);
      atomicExch(p.done_counter, 0);
    }
  }
}

}  // namespace hstu
