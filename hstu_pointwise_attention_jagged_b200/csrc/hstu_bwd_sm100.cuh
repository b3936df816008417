// hstu_bwd_sm100.cuh — backward pass of jagged target-aware HSTU pointwise attention for sm_100a.
//
// Forward (DLRMv3 review, section "model selection"): out = Mask(SiLU(alpha Q K^T)) V / N.  The
// pages print no backward pass; by the chain rule, with dO the loss gradient of out and for every
// visible pair (i, j):
//   x = alpha q_i.k_j,  p = silu(x),  g = dO_i.v_j / N,  ds = g silu'(x) alpha
//   dV_j += p dO_i / N,  dQ_i += ds k_j,  dK_j += ds q_i
// With h = x/2 and t = tanh(h):  p = h (1 + t),  silu'(x) = (1 + t)(1 + h - h t) / 2, so one
// tanh.approx.f32 per pair gives both p and silu'.
//
// hstu_bwd_kernel<D, kDQ> is one persistent kernel body for both halves of the work:
//   kDQ = false (dK/dV): an item owns one 128-key tile; its K and V tiles stay in shared memory
//       ("fixed" pair) while the query tiles that see it stream through a ring (Q and dO).
//         S^T = K Q^T, dP^T = V dO^T                      (SS MMAs into TMEM)
//         P^T, dS^T in registers (thread = key row)        -> bf16 into TMEM over S^T, dP^T
//         dV += P^T dO, dK += dS^T Q                       (TS MMAs, P^T / dS^T read from TMEM)
//   kDQ = true (dQ): an item owns one 128-query tile; Q and dO stay, K and V stream.
//         S = Q K^T, dP = dO V^T;  dS (thread = query row);  dQ += dS K
// No atomics: every output row is written once, by the item that owns it.
//
//   warp 8      producer: fetches the next item, TMA-loads the fixed pair and streams the pairs
//   warp 9      MMA issuer (lane 0 issues, the warp runs converged)
//   warps 0-7   elementwise + epilogue: warp w owns TMEM lane quarter w % 4 and score columns
//               [64 (w / 4), 64 (w / 4) + 64); its bf16 results overwrite the first half of its
//               own column range, so no warp writes a column another warp still has to read.
//
// TMEM columns: S [0,128), dP [128,256), accumulator 0 [256, 256+D), accumulator 1 [256+D, 256+2D)
// (dK/dV: acc0 = dV, acc1 = dK;  dQ: acc0 = dQ).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "bwd_schedule.cuh"
#include "hstu_fwd_sm100.cuh"
#include "sm100_ptx.cuh"

namespace hstu {

template <int D>
struct BwdCfg {
  using T = FwdCfg<D>;  // tile geometry: swizzle, column blocks, bytes per 128-row tile
  static constexpr int kStages = (D == 128) ? 2 : 4;  // ring stages; each holds a pair of tiles
  static constexpr int kSmemTiles = (2 + 2 * kStages) * T::kTileBytes;
  static constexpr int kSmemBytes = 1024 + kSmemTiles + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0, kColDP = 128, kColA0 = 256, kColA1 = 256 + D;
  static constexpr uint32_t kIdescScore = ptx::idesc_bf16_f32(128, 128, false);
  static constexpr uint32_t kIdescAcc = ptx::idesc_bf16_f32(128, D, true);
};

constexpr int kBwdThreads = 320;

struct BwdParams {
  const int32_t* seq_offsets;
  const int32_t* num_targets;  // may be null
  const int4* items;
  const int32_t* num_items;
  int32_t* work_counter;
  int32_t* done_counter;
  __nv_bfloat16* out0;  // dK/dV: dV;  dQ: dQ
  __nv_bfloat16* out1;  // dK/dV: dK;  dQ: unused
  int32_t H;
  float half_alpha;     // alpha / 2
  float ds_scale;       // alpha / (2 N)
  float inv_n;
  unsigned* err;
  // dK/dV kernel, when the dQ pass reads dS instead of recomputing it: the dS workspace (ds_cap
  // tiles of 128 x 128 bf16, row-major [key][query]) and each user's first tile (plan).
  __nv_bfloat16* ds_ws;
  const long long* ds_base;
  long long ds_cap;
};

template <int kStages>
struct BwdCtl {
  uint64_t fix_full, fix_empty;
  uint64_t ring_full[kStages], ring_empty[kStages];
  // s_full / dp_full: the score MMAs of a tile committed; p_full: the elementwise warps are done with
  // S (dK/dV: P written; dQ: S read); ds_full: dS written.
  uint64_t s_full, dp_full, p_full, ds_full, o_full, o_empty;
  uint64_t sched_full[2], sched_empty[2];
  uint64_t drain;
  // work slot: valid, h, row0 (first token row of the user), fixed tile, L, U, e1, s2, e2
  int32_t slot[2][10];
  uint32_t tmem_base;
  int32_t abort_flag;
};

struct BwdWork {
  int valid, h, row0, fixed, L, U;
  TileRange r;
  int b;
};

__device__ __forceinline__ BwdWork read_bwd_slot(const volatile int32_t* s) {
  BwdWork w;
  w.valid = s[0];
  w.h = s[1];
  w.row0 = s[2];
  w.fixed = s[3];
  w.L = s[4];
  w.U = s[5];
  w.r.e1 = s[6];
  w.r.s2 = s[7];
  w.r.e2 = s[8];
  w.b = s[9];
  return w;
}

// First half of the elementwise step, 32 score columns of this thread's row.  From S it forms the
// SiLU factor m = (1 + t)(1 + h - h t) of every column, kept in registers for the second half, and
// (dK/dV) P = h (1 + t), packed as bf16 pairs into 16 TMEM columns.  The visible columns are
// [lo, hi) plus `self` (relative to the chunk's first column); P is an exact zero elsewhere.
// Columns go in pairs on the two-wide FMA pipe.  kMasked = false is the form for a warp whose 32
// rows see all 64 columns: it carries no per-column tests.
template <bool kDQ, bool kMasked>
__device__ __forceinline__ void bwd_scores(const uint32_t (&s)[32], float (&m)[32], uint32_t t_p, float half_alpha,
                                           int lo, int hi, int self) {
  uint32_t pk_p[16];
  const uint64_t ha2 = ptx::f32x2(half_alpha, half_alpha);
  const uint64_t one2 = ptx::f32x2(1.0f, 1.0f);
  const uint64_t neg2 = ptx::f32x2(-1.0f, -1.0f);
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const int c = 2 * e;
    const uint64_t h2 = ptx::mul_f32x2(ptx::f32x2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), ha2);
    float h0, h1;
    ptx::f32x2_split(h2, h0, h1);
    const uint64_t t2 = ptx::f32x2(ptx::tanh_approx(h0), ptx::tanh_approx(h1));
    const uint64_t a2 = ptx::fma_f32x2(t2, one2, one2);  // 1 + t
    const uint64_t p2 = ptx::mul_f32x2(h2, a2);          // p = h (1 + t)
    // m = (1 + t)(1 + h - h t) = (1 + t) + p (1 - t)
    ptx::f32x2_split(ptx::fma_f32x2(p2, ptx::fma_f32x2(t2, neg2, one2), a2), m[c], m[c + 1]);
    if constexpr (!kDQ) {
      float p0, p1;
      ptx::f32x2_split(p2, p0, p1);
      if constexpr (kMasked) {
        p0 = ((c >= lo && c < hi) || c == self) ? p0 : 0.0f;
        p1 = ((c + 1 >= lo && c + 1 < hi) || c + 1 == self) ? p1 : 0.0f;
      }
      pk_p[e] = pack_bf16x2(p0, p1);
    }
  }
  if constexpr (!kDQ) ptx::tmem_st16(t_p, pk_p);
}

// Second half: dS = (dP ds_scale) m, an exact zero outside the visible columns, packed as bf16
// pairs into 16 TMEM columns.
template <bool kMasked>
__device__ __forceinline__ void bwd_grads(const uint32_t (&dp)[32], const float (&m)[32], uint32_t t_ds,
                                          float ds_scale, int lo, int hi, int self, uint4* g_ds) {
  uint32_t pk[16];
  const uint64_t sc2 = ptx::f32x2(ds_scale, ds_scale);
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const int c = 2 * e;
    float d0, d1;
    ptx::f32x2_split(ptx::mul_f32x2(ptx::mul_f32x2(ptx::f32x2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])), sc2),
                                    ptx::f32x2(m[c], m[c + 1])),
                     d0, d1);
    if constexpr (kMasked) {
      d0 = ((c >= lo && c < hi) || c == self) ? d0 : 0.0f;
      d1 = ((c + 1 >= lo && c + 1 < hi) || c + 1 == self) ? d1 : 0.0f;
    }
    pk[e] = pack_bf16x2(d0, d1);
  }
  ptx::tmem_st16(t_ds, pk);
  if (g_ds != nullptr) {
    // The same 32 values into the dS workspace for the dQ pass (written once, read by another
    // kernel): 64 bytes, 32-byte aligned, as two whole-sector stores.
#pragma unroll
    for (int h = 0; h < 2; ++h)
      asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(g_ds + 2 * h),
                   "r"(pk[8 * h]), "r"(pk[8 * h + 1]), "r"(pk[8 * h + 2]), "r"(pk[8 * h + 3]), "r"(pk[8 * h + 4]),
                   "r"(pk[8 * h + 5]), "r"(pk[8 * h + 6]), "r"(pk[8 * h + 7])
                   : "memory");
  }
}

template <int D, bool kDQ>
__global__ void __launch_bounds__(kBwdThreads, 1)
    hstu_bwd_kernel(const __grid_constant__ CUtensorMap tm_f0, const __grid_constant__ CUtensorMap tm_f1,
                    const __grid_constant__ CUtensorMap tm_s0, const __grid_constant__ CUtensorMap tm_s1,
                    const BwdParams p) {
  using Cfg = BwdCfg<D>;
  using T = typename Cfg::T;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  const uint32_t sbase = ptx::smem_addr(smem);
  const uint32_t sFix = sbase;                          // 2 tiles: fixed[0], fixed[1]
  const uint32_t sRing = sbase + 2 * T::kTileBytes;     // kStages x 2 tiles
  auto* ctl = reinterpret_cast<BwdCtl<Cfg::kStages>*>(smem + Cfg::kSmemTiles);
  volatile int32_t* abort_flag = &ctl->abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  auto bar = [](const uint64_t& b) { return ptx::smem_addr(&b); };

  if (warp == kProducerWarp && lane == 0) {
    ptx::mbar_init(bar(ctl->fix_full), 1);
    ptx::mbar_init(bar(ctl->fix_empty), 1);
    for (int s = 0; s < Cfg::kStages; ++s) {
      ptx::mbar_init(bar(ctl->ring_full[s]), 1);
      ptx::mbar_init(bar(ctl->ring_empty[s]), 1);
    }
    ptx::mbar_init(bar(ctl->s_full), 1);
    ptx::mbar_init(bar(ctl->dp_full), 1);
    ptx::mbar_init(bar(ctl->p_full), 8);
    ptx::mbar_init(bar(ctl->ds_full), 8);
    ptx::mbar_init(bar(ctl->o_full), 1);
    ptx::mbar_init(bar(ctl->o_empty), 8);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar(ctl->sched_full[i]), 1);
      ptx::mbar_init(bar(ctl->sched_empty[i]), 1 + 8);
    }
    ptx::mbar_init(bar(ctl->drain), 1);
    ctl->abort_flag = 0;
    ptx::fence_mbarrier_init();
    ptx::prefetch_tmap(&tm_f0);
    ptx::prefetch_tmap(&tm_f1);
    ptx::prefetch_tmap(&tm_s0);
    ptx::prefetch_tmap(&tm_s1);
  }
  if (warp == kMmaWarp) {
    ptx::tmem_alloc(ptx::smem_addr(&ctl->tmem_base), Cfg::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      asm volatile("griddepcontrol.wait;" ::: "memory");
      const int M = *p.num_items;
      int slot = 0;
      uint32_t sched_empty_par[2] = {1u, 1u};
      uint32_t fix_empty_par = 1u;
      int stage = 0;
      uint32_t ring_phase = 0;
      bool ok = true;
      int issued_fix = 0, issued_ring = 0;
      while (ok) {
        const int idx = atomicAdd(p.work_counter, 1);
        BwdWork w{};
        w.valid = idx < M;
        if (w.valid) {
          const int4 it = p.items[idx];
          const int b = it.x;
          w.b = b;
          w.fixed = it.y;
          w.h = it.z;
          w.row0 = p.seq_offsets[b];
          w.L = p.seq_offsets[b + 1] - w.row0;
          w.U = w.L - (p.num_targets ? p.num_targets[b] : 0);
          w.r = kDQ ? key_tiles_of_query_tile(w.fixed, w.L, w.U) : query_tiles_of_key_tile(w.fixed, w.L, w.U);
        }
        if (!wait_bounded(bar(ctl->sched_empty[slot]), sched_empty_par[slot], abort_flag, p.err)) break;
        sched_empty_par[slot] ^= 1u;
        volatile int32_t* s = ctl->slot[slot];
        s[0] = w.valid; s[1] = w.h; s[2] = w.row0; s[3] = w.fixed; s[4] = w.L; s[5] = w.U;
        s[6] = w.r.e1; s[7] = w.r.s2; s[8] = w.r.e2; s[9] = w.b;
        ptx::mbar_arrive(bar(ctl->sched_full[slot]));
        slot ^= 1;
        if (!w.valid) break;

        const int col = w.h * D;
        if (!wait_bounded(bar(ctl->fix_empty), fix_empty_par, abort_flag, p.err)) break;
        fix_empty_par ^= 1u;
        ptx::mbar_arrive_expect_tx(bar(ctl->fix_full), 2 * T::kTileBytes);
        for (int blk = 0; blk < T::kBlocks; ++blk) {
          const int row = w.row0 + w.fixed * kTileRows;
          ptx::tma_load_2d(sFix + blk * T::kBlockBytes, &tm_f0, bar(ctl->fix_full), col + blk * T::kBlockElems, row);
          ptx::tma_load_2d(sFix + T::kTileBytes + blk * T::kBlockBytes, &tm_f1, bar(ctl->fix_full),
                           col + blk * T::kBlockElems, row);
        }
        ++issued_fix;
        const int n = tile_count(w.r);
        for (int i = 0; i < n; ++i) {
          if (!wait_bounded(bar(ctl->ring_empty[stage]), ring_phase ^ 1u, abort_flag, p.err)) {
            ok = false;
            break;
          }
          const uint32_t fb = bar(ctl->ring_full[stage]);
          ptx::mbar_arrive_expect_tx(fb, 2 * T::kTileBytes);
          const int row = w.row0 + tile_at(w.r, i) * kTileRows;
          const uint32_t dst = sRing + stage * 2 * T::kTileBytes;
          for (int blk = 0; blk < T::kBlocks; ++blk) {
            ptx::tma_load_2d(dst + blk * T::kBlockBytes, &tm_s0, fb, col + blk * T::kBlockElems, row);
            ptx::tma_load_2d(dst + T::kTileBytes + blk * T::kBlockBytes, &tm_s1, fb, col + blk * T::kBlockElems, row);
          }
          ++issued_ring;
          if (++stage == Cfg::kStages) {
            stage = 0;
            ring_phase ^= 1u;
          }
        }
      }
      if (*abort_flag) {
        // Let every copy this CTA started land before its shared memory is released.
        for (int k = 1; k <= Cfg::kStages && k <= issued_ring; ++k) {
          const int pos = issued_ring - k;
          drain_wait(bar(ctl->ring_full[pos % Cfg::kStages]), (uint32_t)((pos / Cfg::kStages) & 1));
        }
        if (issued_fix > 0) drain_wait(bar(ctl->fix_full), (uint32_t)((issued_fix - 1) & 1));
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    const uint32_t lead = (lane == 0) ? 1u : 0u;
    auto wait_all = [&](uint32_t b, uint32_t par) {
      return __all_sync(0xffffffffu, wait_bounded(b, par, abort_flag, p.err));
    };
    const uint64_t dfix = ptx::smem_desc(sFix, 16, 8 * T::kRowBytes, T::kSwizzle);       // K-major A
    const uint64_t dring = ptx::smem_desc(sRing, 16, 8 * T::kRowBytes, T::kSwizzle);     // K-major B
    const uint64_t dringmn = ptx::smem_desc(sRing, T::kBlockBytes, 8 * T::kRowBytes, T::kSwizzle);  // MN-major B
    int slot = 0;
    uint32_t sched_full_par[2] = {0u, 0u};
    uint32_t fix_full_par = 0u, p_full_par = 0u, ds_full_par = 0u, o_empty_par = 1u;
    int stage = 0;
    uint32_t ring_phase = 0;
    bool ok = true;
    // Score MMAs of the streamed tile in ring stage `sst`: which = 0 gives S (fixed[0] x
    // streamed[0]^T), which = 1 gives dP (fixed[1] x streamed[1]^T).
    auto scores = [&](int sst, int which) {
      const uint64_t dst = dring + ((sst * 2 * T::kTileBytes + which * T::kTileBytes) >> 4);
      const uint64_t dfx = dfix + ((which * T::kTileBytes) >> 4);
      const uint32_t col = which ? Cfg::kColDP : Cfg::kColS;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t off = (ks / T::kKStepsPerBlock) * T::kBlockBytes + (ks % T::kKStepsPerBlock) * 32;
        ptx::mma_ss_lead(lead, tmem + col, dfx + (off >> 4), dst + (off >> 4), Cfg::kIdescScore, ks > 0 ? 1u : 0u);
      }
    };
    // acc += A B with A (bf16 P or dS) read from TMEM at column a_col and B the streamed tile `which`
    // of ring stage `sst` (MN-major); `first` starts the accumulator afresh.
    auto accum = [&](int sst, uint32_t acc_col, uint32_t a_col, int which, bool first) {
      const uint64_t dmn = dringmn + ((sst * 2 * T::kTileBytes + which * T::kTileBytes) >> 4);
#pragma unroll
      for (int ks = 0; ks < kTileRows / 16; ++ks) {
        const uint32_t acol = 64 * (ks >> 2) + 8 * (ks & 3);
        ptx::mma_ts_lead(lead, tmem + acc_col, tmem + a_col + acol, dmn + ((ks * 16 * T::kRowBytes) >> 4),
                         Cfg::kIdescAcc, (first && ks == 0) ? 0u : 1u);
      }
    };
    auto next_stage = [&]() {
      if (++stage == Cfg::kStages) {
        stage = 0;
        ring_phase ^= 1u;
      }
    };
    while (ok) {
      if (!wait_all(bar(ctl->sched_full[slot]), sched_full_par[slot])) break;
      sched_full_par[slot] ^= 1u;
      const BwdWork w = read_bwd_slot(ctl->slot[slot]);
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(ctl->sched_empty[slot]));
      slot ^= 1;
      if (!w.valid) break;
      const int n = tile_count(w.r);
      if (!wait_all(bar(ctl->fix_full), fix_full_par)) break;
      fix_full_par ^= 1u;
      // Tile 0's scores.
      int cur = stage;
      if (n > 0) {
        if (!wait_all(bar(ctl->ring_full[stage]), ring_phase)) break;
        next_stage();
        ptx::tc_fence_after();
        scores(cur, 0);
        ptx::mma_commit_lead(lead, bar(ctl->s_full));
        scores(cur, 1);
        ptx::mma_commit_lead(lead, bar(ctl->dp_full));
      }
      // Tile i's gradient MMAs wait for its elementwise halves; tile i+1's score MMAs fill the gaps.
      //   dK/dV:  dV(i) [P_i]  S(i+1)  dK(i) [dS_i]  dP(i+1)
      //   dQ:     S(i+1) [S_i read]  dQ(i) [dS_i]  dP(i+1)
      // Every overwrite of a TMEM buffer is issued after the MMA that last reads it (tcgen05 MMAs of
      // one thread run in order), and after the elementwise warps have released it.
      for (int i = 0; i < n && ok; ++i) {
        const bool more = i + 1 < n;
        const int nxt = stage;
        const uint32_t nph = ring_phase;
        if (more) next_stage();
        ok = wait_all(bar(ctl->p_full), p_full_par);
        if (!ok) break;
        p_full_par ^= 1u;
        if constexpr (!kDQ) {
          if (i == 0) {
            if (!wait_all(bar(ctl->o_empty), o_empty_par)) { ok = false; break; }
            o_empty_par ^= 1u;
          }
          ptx::tc_fence_after();
          accum(cur, Cfg::kColA0, Cfg::kColS, 1, i == 0);  // dV += P^T dO
        }
        if (more) {
          if (!wait_all(bar(ctl->ring_full[nxt]), nph)) { ok = false; break; }
          ptx::tc_fence_after();
          scores(nxt, 0);
          ptx::mma_commit_lead(lead, bar(ctl->s_full));
        }
        if (!wait_all(bar(ctl->ds_full), ds_full_par)) { ok = false; break; }
        ds_full_par ^= 1u;
        if constexpr (kDQ) {
          if (i == 0) {
            if (!wait_all(bar(ctl->o_empty), o_empty_par)) { ok = false; break; }
            o_empty_par ^= 1u;
          }
        }
        ptx::tc_fence_after();
        if constexpr (kDQ) accum(cur, Cfg::kColA0, Cfg::kColDP, 0, i == 0);  // dQ += dS K
        else accum(cur, Cfg::kColA1, Cfg::kColDP, 0, i == 0);                // dK += dS^T Q
        ptx::mma_commit_lead(lead, bar(ctl->ring_empty[cur]));  // tile i's streamed pair is done
        if (more) {
          scores(nxt, 1);
          ptx::mma_commit_lead(lead, bar(ctl->dp_full));
        }
        cur = nxt;
      }
      if (!ok) break;
      ptx::mma_commit_lead(lead, bar(ctl->fix_empty));  // fixed pair free after the item's last MMA
      ptx::mma_commit_lead(lead, bar(ctl->o_full));     // accumulators complete
    }
    ptx::mma_commit_lead(lead, bar(ctl->drain));
    drain_wait(bar(ctl->drain), 0u);
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ elementwise + epilogue
    const int quarter = warp & 3;
    const int ch = warp >> 2;                      // score columns [64 ch, 64 ch + 64)
    const int row = quarter * 32 + lane;           // row of the fixed tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t t_s = tmem + lane_off + Cfg::kColS + 64 * ch;
    const uint32_t t_dp = tmem + lane_off + Cfg::kColDP + 64 * ch;
    int slot = 0;
    uint32_t sched_full_par[2] = {0u, 0u};
    uint32_t s_full_par = 0u, dp_full_par = 0u, o_full_par = 0u;
    bool ok = true;
    while (ok) {
      ok = __all_sync(0xffffffffu, wait_bounded(bar(ctl->sched_full[slot]), sched_full_par[slot], abort_flag, p.err));
      if (!ok) break;
      sched_full_par[slot] ^= 1u;
      const BwdWork w = read_bwd_slot(ctl->slot[slot]);
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(ctl->sched_empty[slot]));
      slot ^= 1;
      if (!w.valid) break;
      const int n = tile_count(w.r);
      const int pos = w.fixed * kTileRows + row;  // this thread's position in the segment
      for (int i = 0; i < n; ++i) {
        const int c0 = tile_at(w.r, i) * kTileRows + 64 * ch;  // position of this warp's first column
        ok = __all_sync(0xffffffffu, wait_bounded(bar(ctl->s_full), s_full_par, abort_flag, p.err));
        if (!ok) break;
        s_full_par ^= 1u;
        ptx::tc_fence_after();
        // Visible columns, relative to c0: [lo, hi) plus self.
        int lo, hi, self;
        bool full;
        if constexpr (kDQ) {
          // query `pos` sees keys [0, min(pos + 1, U)) and itself
          lo = -c0;
          hi = (pos < w.U ? pos + 1 : w.U) - c0;
          self = pos - c0;
          full = (c0 + 64 <= w.U) && (c0 + 64 <= pos + 1) && pos < w.L;
        } else {
          // key `pos` is seen by queries [pos, L) if it is history, by itself alone otherwise
          lo = pos - c0;
          hi = (pos < w.U ? w.L : pos + 1) - c0;
          if (pos >= w.L) hi = lo;
          self = -1;
          full = (lo <= 0) && (hi >= 64);
        }
        // The mask-free forms run only when every row of the warp sees all 64 columns, so the warp
        // takes one branch.
        full = __all_sync(0xffffffffu, full);
        // First half: S -> the SiLU factors (registers) and, for dK/dV, P over S.  Then S is released.
        float m[2][32];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          uint32_t rs[32];
          ptx::tmem_ld32(t_s + 32 * k, rs);
          ptx::tmem_ld_wait(rs);
          if (full)
            bwd_scores<kDQ, false>(rs, m[k], t_s + 16 * k, p.half_alpha, lo - 32 * k, hi - 32 * k, self - 32 * k);
          else
            bwd_scores<kDQ, true>(rs, m[k], t_s + 16 * k, p.half_alpha, lo - 32 * k, hi - 32 * k, self - 32 * k);
        }
        if constexpr (!kDQ) ptx::tmem_st_wait();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(ctl->p_full));
        // Second half: dP -> dS over dP (and, for the dQ pass, into the workspace: tile (key tile
        // w.fixed, query tile w.fixed + i) of this user and head, this thread's row and 64 columns).
        uint4* g_ds = nullptr;
        if constexpr (!kDQ) {
          if (p.ds_ws != nullptr) {
            const long long tile = p.ds_base[w.b] + (long long)w.h * ds_tiles_per_head(w.L, w.U) +
                                   ds_tiles_before(w.fixed, w.L, w.U) + i;
            if (tile < p.ds_cap)
              g_ds = reinterpret_cast<uint4*>(p.ds_ws + (tile * kTileRows + row) * kTileRows + 64 * ch);
            else if (lane == 0)
              atomicOr(p.err, kErrBadOffsets);  // the workspace bound was wrong: report, write nothing
          }
        }
        ok = __all_sync(0xffffffffu, wait_bounded(bar(ctl->dp_full), dp_full_par, abort_flag, p.err));
        if (!ok) break;
        dp_full_par ^= 1u;
        ptx::tc_fence_after();
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          uint32_t rd[32];
          ptx::tmem_ld32(t_dp + 32 * k, rd);
          ptx::tmem_ld_wait(rd);
          if (full)
            bwd_grads<false>(rd, m[k], t_dp + 16 * k, p.ds_scale, lo - 32 * k, hi - 32 * k, self - 32 * k,
                             g_ds ? g_ds + 4 * k : nullptr);
          else
            bwd_grads<true>(rd, m[k], t_dp + 16 * k, p.ds_scale, lo - 32 * k, hi - 32 * k, self - 32 * k,
                            g_ds ? g_ds + 4 * k : nullptr);
        }
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(ctl->ds_full));
      }
      if (!ok) break;
      ok = __all_sync(0xffffffffu, wait_bounded(bar(ctl->o_full), o_full_par, abort_flag, p.err));
      if (!ok) break;
      o_full_par ^= 1u;
      ptx::tc_fence_after();
      // Epilogue: rows of the fixed tile that exist.  dK/dV: warps of column half 0 write dV
      // (scaled by 1/N), half 1 writes dK.  dQ: the two halves split dQ's columns.
      const bool live = w.fixed * kTileRows + row < w.L;
      const size_t grow = (size_t)(w.row0 + w.fixed * kTileRows + row);
      if constexpr (kDQ) {
        constexpr int kPer = (D / 32 + 1) / 2;  // 32-column chunks per warp
#pragma unroll
        for (int c = 0; c < kPer; ++c) {
          const int cc = ch * kPer + c;
          if (cc < D / 32) {
            uint32_t ro[32];
            ptx::tmem_ld32(tmem + lane_off + Cfg::kColA0 + 32 * cc, ro);
            ptx::tmem_ld_wait(ro);
            if (live) {
              uint4* d4 = reinterpret_cast<uint4*>(p.out0 + (grow * p.H + w.h) * D + 32 * cc);
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
        }
      } else {
        const uint32_t col = ch ? Cfg::kColA1 : Cfg::kColA0;
        const float scale = ch ? 1.0f : p.inv_n;
        __nv_bfloat16* dst = (ch ? p.out1 : p.out0) + (grow * p.H + w.h) * D;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t ro[32];
          ptx::tmem_ld32(tmem + lane_off + col + 32 * cc, ro);
          ptx::tmem_ld_wait(ro);
          if (live) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * cc);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              uint4 v;
              v.x = pack_bf16x2(__uint_as_float(ro[q4 * 8 + 0]) * scale, __uint_as_float(ro[q4 * 8 + 1]) * scale);
              v.y = pack_bf16x2(__uint_as_float(ro[q4 * 8 + 2]) * scale, __uint_as_float(ro[q4 * 8 + 3]) * scale);
              v.z = pack_bf16x2(__uint_as_float(ro[q4 * 8 + 4]) * scale, __uint_as_float(ro[q4 * 8 + 5]) * scale);
              v.w = pack_bf16x2(__uint_as_float(ro[q4 * 8 + 6]) * scale, __uint_as_float(ro[q4 * 8 + 7]) * scale);
              d4[q4] = v;
            }
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(ctl->o_empty));
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == kMmaWarp) ptx::tmem_dealloc(tmem, Cfg::kTmemCols);
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.done_counter, 1) == (int)gridDim.x - 1) {
      atomicExch(p.work_counter, 0);
      atomicExch(p.done_counter, 0);
    }
  }
}

}  // namespace hstu
