// hstu_fwd_sm100.cuh — fused forward kernel of jagged target-aware HSTU pointwise attention for
// sm_100a:  out = Mask(SiLU(alpha * Q K^T)) V / N   (DLRMv3 review, section "model selection").
//
// One persistent CTA per SM pulls work items (user b, head h, 256 query rows) from a cost-
// ordered list through an atomic counter.  Per item the two 128-row halves share every K/V tile.
//
//   warp 8      producer: fetches the next item, TMA-loads Q (both halves) and the item's key
//               tiles K_t, V_t into a ring of shared-memory stages (128B/64B swizzle).
//   warp 9      MMA issuer: the warp runs converged and lane 0 issues every tcgen05 instruction.
//               S_h = Q_h K_t^T into TMEM (SS form), then, once the SiLU warps have written P_h,
//               O_h += P_h V_t with P_h read from TMEM (TS form).  Issue order per key tile:
//               PV_0(prev) S_0(t) PV_1(prev) S_1(t), so the tensor core has the other half's work
//               while one half's SiLU runs.
//   warps 0-3   SiLU warpgroup of half 0, warps 4-7 of half 1: TMEM -> registers, p =
//               mask ? silu(alpha*s) : 0 with silu(x) = h + h*tanh(h), h = x/2 (one MUFU op per
//               score), packed to bf16 and written back over S in TMEM; after the item's last
//               tile, the epilogue: O * (1/N) -> bf16 -> row-predicated global stores.
//
// TMEM (512 columns x 128 lanes of fp32): S_0 [0,128), S_1 [128,256), O_0 [256,256+D),
// O_1 [256+D, 256+2D).  P_h (bf16 pairs) overwrites the first 64 columns of S_h.
//
// hstu_fwd_kernel<D, true> is the relative-attention-bias variant: each visible pair's p also gets
// a per-head table entry for its query-key distance (the table is read through the read-only
// cache); everything else is the same kernel.
//
// Every mbarrier wait is bounded by %globaltimer; on expiry the kernel records kErrTimeout,
// raises a CTA-wide abort flag, lets every role leave its loop, drains the copies and MMAs it
// issued, frees TMEM and returns.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "schedule.cuh"
#include "sm100_ptx.cuh"

namespace hstu {

template <int D>
struct FwdCfg {
  static_assert(D == 32 || D == 64 || D == 128, "head size");
  static constexpr int kRowBytes = (D >= 64) ? 128 : 64;  // bytes per swizzled row
  static constexpr int kBlockElems = kRowBytes / 2;       // bf16 per row of one column block
  static constexpr int kBlocks = D / kBlockElems;         // column blocks per tile
  static constexpr int kBlockBytes = kTileRows * kRowBytes;
  static constexpr int kTileBytes = kBlocks * kBlockBytes;  // 128 rows x D bf16
  static constexpr uint32_t kSwizzle = (kRowBytes == 128) ? 2u : 4u;  // UMMA layout code
  static constexpr int kKStepsPerBlock = kBlockElems / 16;
  static constexpr int kStages = (D == 128) ? 4 : 8;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 256 + D;
  static constexpr int kSmemTiles = (2 + kStages) * kTileBytes;
  static constexpr int kSmemBytesRaw = 1024 + kSmemTiles + 1024;
  // Keep one CTA per SM so that the 512-column TMEM allocation never waits on a sibling CTA.
  static constexpr int kSmemBytes = kSmemBytesRaw > 120 * 1024 ? kSmemBytesRaw : 120 * 1024;
  static constexpr uint32_t kIdescQK = ptx::idesc_bf16_f32(128, 128, false);
  static constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(128, D, true);
};

constexpr int kNumThreads = 320;  // 8 SiLU warps + producer + MMA issuer
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;       // issues every MMA and owns the TMEM allocation
constexpr uint64_t kWaitLimitNs = 4000000000ull;  // 4 s per wait
constexpr uint64_t kDrainLimitNs = 200000000ull;  // 0.2 s per drain wait on the abort path

struct FwdParams {
  const int32_t* seq_offsets;
  const int32_t* num_targets;  // may be null
  const int32_t* cached_len;   // may be null
  const int32_t* q_start;      // from the schedule kernel
  const int4* items;
  const int32_t* num_items;
  int32_t* work_counter;
  int32_t* done_counter;
  __nv_bfloat16* out;
  int64_t out_ld;              // elements between consecutive rows of out (H*D when packed)
  // Layer epilogue (all null outside a layer): with gate = U, also writes U to gate_copy and
  // U * A (A rounded to bf16 first) to gate_prod, rows strided like out; U rows are gate_ld apart.
  const __nv_bfloat16* gate;
  int64_t gate_ld;
  __nv_bfloat16* gate_copy;
  __nv_bfloat16* gate_prod;
  const float* rab;            // relative-bias variant: [H, rab_len] table; unused otherwise
  int32_t rab_len;
  int32_t H;
  float half_alpha;
  float inv_n;
  unsigned* err;
  uint64_t wait_limit_ns;      // limit of every pipeline wait (kWaitLimitNs; a self-check lowers it)
};

template <int kStages>
struct SmemCtl {
  uint64_t q_full, q_empty;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], p_full[2], o_full[2], o_empty[2];
  uint64_t sched_full[2], sched_empty[2];
  uint64_t drain;
  // work slot: valid, h, kv_start, q_row0, pos0, nrows, L, U
  int32_t slot[2][8];
  uint32_t tmem_base;
  int32_t abort_flag;
};

struct Work {
  int valid, h, kv_start, q_row0, pos0, nrows, L, U;
};

__device__ __forceinline__ Work read_slot(const volatile int32_t* s) {
  Work w;
  w.valid = s[0];
  w.h = s[1];
  w.kv_start = s[2];
  w.q_row0 = s[3];
  w.pos0 = s[4];
  w.nrows = s[5];
  w.L = s[6];
  w.U = s[7];
  return w;
}

// Slow path of wait_bounded: spins until the phase completes, the CTA aborts, or the time limit.
// Each try_wait may itself suspend the thread for a while, so the flag and the clock are checked
// after every attempt.
__device__ __noinline__ bool wait_bounded_slow(uint32_t bar, uint32_t parity, volatile int32_t* abort_flag,
                                               unsigned* err, uint64_t limit_ns) {
  const uint64_t t0 = ptx::globaltimer_ns();
  while (true) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (ptx::globaltimer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicOr(err, kErrTimeout);
      return false;
    }
  }
}

// Waits for phase `parity` of `bar`; false if the CTA is aborting or this wait timed out.  The
// first test is inline: a call right after a burst of MMAs stalls the issuing warp.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int32_t* abort_flag,
                                             unsigned* err, uint64_t limit_ns = kWaitLimitNs) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  return wait_bounded_slow(bar, parity, abort_flag, err, limit_ns);
}

// Abort-path drain: waits for phase `parity` of `bar` for at most kDrainLimitNs.
__device__ __noinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = ptx::globaltimer_ns();
  while (!ptx::mbar_try_wait(bar, parity))
    if (ptx::globaltimer_ns() - t0 > kDrainLimitNs) return;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Elementwise product of two bf16 pairs, each product formed in fp32 and rounded to bf16 once.
__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
  const float a0 = __uint_as_float(a << 16), a1 = __uint_as_float(a & 0xffff0000u);
  const float b0 = __uint_as_float(b << 16), b1 = __uint_as_float(b & 0xffff0000u);
  return pack_bf16x2(a0 * b0, a1 * b1);
}

// SiLU + mask + bf16 pack of 32 score columns [32*chunk, 32*chunk+32) of this thread's row,
// written as 16 packed columns [16*chunk, 16*chunk+16) of the same TMEM row.
// lim/self are relative to the tile's first key: key column c is visible iff c < lim || c == self.
// With kRab, a visible pair also gets rab_row[min(rel0 - c, rab_max)], its query-key distance
// clipped to the last table entry (rel0 = query position - first key of the tile).
template <int kChunk, bool kRab>
__device__ __forceinline__ void silu_chunk(const uint32_t (&r)[32], uint32_t taddr_s, float half_alpha,
                                           bool full, int lim, int self, const float* rab_row, int rel0,
                                           int rab_max) {
  uint32_t pk[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const float h0 = __uint_as_float(r[2 * e]) * half_alpha;
    const float h1 = __uint_as_float(r[2 * e + 1]) * half_alpha;
    float p0 = fmaf(h0, ptx::tanh_approx(h0), h0);
    float p1 = fmaf(h1, ptx::tanh_approx(h1), h1);
    if constexpr (kRab) {
      // The chunk's distances run down from hi = rel0 - 32*chunk by one per column.  Inside the
      // table the reads are fixed offsets from one base; otherwise (masked pairs have negative
      // distances, far pairs exceed the table) each index is clamped into it.
      const int hi = rel0 - kChunk * 32;
      if (hi >= 31 && hi <= rab_max) {
        p0 += __ldg(rab_row + hi - 2 * e);
        p1 += __ldg(rab_row + hi - 2 * e - 1);
      } else {
        p0 += __ldg(rab_row + min(max(hi - 2 * e, 0), rab_max));
        p1 += __ldg(rab_row + min(max(hi - 2 * e - 1, 0), rab_max));
      }
    }
    if (!full) {
      const int c0 = kChunk * 32 + 2 * e;
      p0 = (c0 < lim || c0 == self) ? p0 : 0.0f;
      p1 = (c0 + 1 < lim || c0 + 1 == self) ? p1 : 0.0f;
    }
    pk[e] = pack_bf16x2(p0, p1);
  }
  ptx::tmem_st16(taddr_s + kChunk * 16, pk);
}

template <int D, bool kRab>
__global__ void __launch_bounds__(kNumThreads, 1)
    hstu_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using Cfg = FwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the 128B-swizzle atoms.
  const uint32_t raw_addr = ptx::smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  const uint32_t sbase = ptx::smem_addr(smem);
  const uint32_t sQ = sbase;                                  // 2 tiles
  const uint32_t sKV = sbase + 2 * Cfg::kTileBytes;           // kStages tiles
  auto* ctl = reinterpret_cast<SmemCtl<Cfg::kStages>*>(smem + Cfg::kSmemTiles);
  volatile int32_t* abort_flag = &ctl->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  auto bar = [](const uint64_t& b) { return ptx::smem_addr(&b); };

  if (warp == kProducerWarp && lane == 0) {
    ptx::mbar_init(bar(ctl->q_full), 1);
    ptx::mbar_init(bar(ctl->q_empty), 1);
    for (int s = 0; s < Cfg::kStages; ++s) {
      ptx::mbar_init(bar(ctl->kv_full[s]), 1);
      ptx::mbar_init(bar(ctl->kv_empty[s]), 1);
    }
    for (int h = 0; h < 2; ++h) {
      ptx::mbar_init(bar(ctl->s_full[h]), 1);
      ptx::mbar_init(bar(ctl->p_full[h]), 4);   // one arrival per SiLU warp
      ptx::mbar_init(bar(ctl->o_full[h]), 1);
      ptx::mbar_init(bar(ctl->o_empty[h]), 4);
      ptx::mbar_init(bar(ctl->sched_full[h]), 1);
      ptx::mbar_init(bar(ctl->sched_empty[h]), 1 + 8);
    }
    ptx::mbar_init(bar(ctl->drain), 1);
    ctl->abort_flag = 0;
    ptx::fence_mbarrier_init();
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_k);
    ptx::prefetch_tmap(&tm_v);
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
      // Everything before this point touched only shared memory, TMEM and kernel parameters; the
      // plan (and q/k/v) come from the preceding grid.
      asm volatile("griddepcontrol.wait;" ::: "memory");
      const int M = *p.num_items;
      int slot = 0;
      uint32_t sched_empty_par[2] = {1u, 1u};
      uint32_t q_empty_par = 1u;
      int stage = 0;
      uint32_t kv_phase = 0;
      bool ok = true;
      int issued_q = 0, issued_kv = 0;
      while (ok) {
        const int idx = atomicAdd(p.work_counter, 1);
        Work w{};
        w.valid = idx < M;
        if (w.valid) {
          const int4 it = p.items[idx];
          const int b = it.x, pair = it.y;
          w.h = it.z;
          w.kv_start = p.seq_offsets[b];
          w.L = p.seq_offsets[b + 1] - w.kv_start;
          const int T = p.num_targets ? p.num_targets[b] : 0;
          const int c = p.cached_len ? p.cached_len[b] : 0;
          w.U = w.L - T;
          w.q_row0 = p.q_start[b] + pair * kPairRows;
          w.pos0 = c + pair * kPairRows;
          const int rows = (w.L - c) - pair * kPairRows;
          w.nrows = rows < kPairRows ? rows : kPairRows;
        }
        if (!wait_bounded(bar(ctl->sched_empty[slot]), sched_empty_par[slot], abort_flag, p.err, p.wait_limit_ns)) break;
        sched_empty_par[slot] ^= 1u;
        volatile int32_t* s = ctl->slot[slot];
        s[0] = w.valid; s[1] = w.h; s[2] = w.kv_start; s[3] = w.q_row0;
        s[4] = w.pos0; s[5] = w.nrows; s[6] = w.L; s[7] = w.U;
        ptx::mbar_arrive(bar(ctl->sched_full[slot]));
        slot ^= 1;
        if (!w.valid) break;

        const TileRange un = key_tiles(w.pos0, w.pos0 + w.nrows, w.U);
        const int n_u = tile_count(un);
        if (!wait_bounded(bar(ctl->q_empty), q_empty_par, abort_flag, p.err, p.wait_limit_ns)) break;
        q_empty_par ^= 1u;
        ptx::mbar_arrive_expect_tx(bar(ctl->q_full), 2 * Cfg::kTileBytes);
        for (int hh = 0; hh < 2; ++hh)
          for (int blk = 0; blk < Cfg::kBlocks; ++blk)
            ptx::tma_load_2d(sQ + hh * Cfg::kTileBytes + blk * Cfg::kBlockBytes, &tm_q, bar(ctl->q_full),
                             w.h * D + blk * Cfg::kBlockElems, w.q_row0 + hh * kTileRows);
        ++issued_q;
        for (int i = 0; i < n_u && ok; ++i) {
          const int row = w.kv_start + tile_at(un, i) * kTileRows;
          for (int kv = 0; kv < 2; ++kv) {
            if (!wait_bounded(bar(ctl->kv_empty[stage]), kv_phase ^ 1u, abort_flag, p.err, p.wait_limit_ns)) {
              ok = false;
              break;
            }
            const uint32_t fb = bar(ctl->kv_full[stage]);
            ptx::mbar_arrive_expect_tx(fb, Cfg::kTileBytes);
            const CUtensorMap* tm = kv ? &tm_v : &tm_k;
            for (int blk = 0; blk < Cfg::kBlocks; ++blk)
              ptx::tma_load_2d(sKV + stage * Cfg::kTileBytes + blk * Cfg::kBlockBytes, tm, fb,
                               w.h * D + blk * Cfg::kBlockElems, row);
            ++issued_kv;
            if (++stage == Cfg::kStages) {
              stage = 0;
              kv_phase ^= 1u;
            }
          }
        }
      }
      if (*abort_flag) {
        // Let every copy this CTA started land before its shared memory is released.
        for (int k = 1; k <= Cfg::kStages && k <= issued_kv; ++k) {
          const int pos = issued_kv - k;  // load index
          drain_wait(bar(ctl->kv_full[pos % Cfg::kStages]), (uint32_t)((pos / Cfg::kStages) & 1));
        }
        if (issued_q > 0) drain_wait(bar(ctl->q_full), (uint32_t)((issued_q - 1) & 1));
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop in step, so the control flow is uniform and the descriptors
    // and TMEM addresses stay in uniform registers; lane 0 alone issues the tcgen05 instructions
    // (the *_lead forms), so every MMA and commit comes from one thread, as commit tracking needs.
    const uint32_t lead = (lane == 0) ? 1u : 0u;
    // Waits are taken by every lane and the outcome is made warp-uniform.
    auto wait_all = [&](uint32_t b, uint32_t par) {
      return __all_sync(0xffffffffu, wait_bounded(b, par, abort_flag, p.err, p.wait_limit_ns));
    };
    // Descriptor templates: the descriptor of address a + off is template(a) + (off >> 4).
    const uint64_t dq0 = ptx::smem_desc(sQ, 16, 8 * Cfg::kRowBytes, Cfg::kSwizzle);
    const uint64_t dk0 = ptx::smem_desc(sKV, 16, 8 * Cfg::kRowBytes, Cfg::kSwizzle);
    const uint64_t dv0 = ptx::smem_desc(sKV, Cfg::kBlockBytes, 8 * Cfg::kRowBytes, Cfg::kSwizzle);
    int slot = 0;
    uint32_t sched_full_par[2] = {0u, 0u};
    uint32_t q_full_par = 0u;
    uint32_t p_full_par[2] = {0u, 0u};
    uint32_t o_empty_par[2] = {1u, 1u};
    int stage = 0;
    uint32_t kv_phase = 0;
    bool ok = true;
    while (ok) {
      if (!wait_all(bar(ctl->sched_full[slot]), sched_full_par[slot])) break;
      sched_full_par[slot] ^= 1u;
      const Work w = read_slot(ctl->slot[slot]);
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(ctl->sched_empty[slot]));
      slot ^= 1;
      if (!w.valid) break;

      const TileRange un = key_tiles(w.pos0, w.pos0 + w.nrows, w.U);
      TileRange hr[2];
      int remaining[2];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int lo = hh * kTileRows;
        const int hi = w.nrows < lo + kTileRows ? w.nrows : lo + kTileRows;
        hr[hh] = key_tiles(w.pos0 + lo, w.pos0 + (hi > lo ? hi : lo), w.U);
        remaining[hh] = tile_count(hr[hh]);
      }
      const int n_u = tile_count(un);
      if (!wait_all(bar(ctl->q_full), q_full_par)) break;
      q_full_par ^= 1u;
      ptx::tc_fence_after();

      bool pend[2] = {false, false};
      bool first[2] = {true, true};
      int prev_vst = 0;
      uint32_t prev_vph = 0;
      // Step i, per half in turn: the P.V of the previous key tile (if that half used it), then
      // the scores of key tile i (if that half needs it).  The tensor pipe therefore alternates
      // [P.V_0, S_0], [P.V_1, S_1], and one half's SiLU overlaps the other half's MMAs.  The
      // extra last step only drains the P.V.
      for (int i = 0; i <= n_u; ++i) {
        const bool last = (i == n_u);
        int t = 0, kst = 0, vst = 0;
        uint32_t kph = 0, vph = 0;
        if (!last) {
          t = tile_at(un, i);
          kst = stage;
          kph = kv_phase;
          if (++stage == Cfg::kStages) { stage = 0; kv_phase ^= 1u; }
          vst = stage;
          vph = kv_phase;
          if (++stage == Cfg::kStages) { stage = 0; kv_phase ^= 1u; }
        }
        bool k_waited = false, v_waited = false;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const uint32_t colS = hh ? Cfg::kColS1 : Cfg::kColS0;
          if (pend[hh]) {
            ok = wait_all(bar(ctl->p_full[hh]), p_full_par[hh]) &&
                 (v_waited || wait_all(bar(ctl->kv_full[prev_vst]), prev_vph)) &&
                 (!first[hh] || wait_all(bar(ctl->o_empty[hh]), o_empty_par[hh]));
            if (!ok) break;
            v_waited = true;
            p_full_par[hh] ^= 1u;
            if (first[hh]) o_empty_par[hh] ^= 1u;
            ptx::tc_fence_after();
            const uint64_t dv = dv0 + ((prev_vst * Cfg::kTileBytes) >> 4);
            const uint32_t colO = hh ? Cfg::kColO1 : Cfg::kColO0;
#pragma unroll
            for (int ks = 0; ks < kTileRows / 16; ++ks)
              ptx::mma_ts_lead(lead, tmem + colO, tmem + colS + ks * 8, dv + ((ks * 16 * Cfg::kRowBytes) >> 4),
                               Cfg::kIdescPV, (first[hh] && ks == 0) ? 0u : 1u);
            first[hh] = false;
            pend[hh] = false;
            if (--remaining[hh] == 0) ptx::mma_commit_lead(lead, bar(ctl->o_full[hh]));
          }
          if (!last && tile_in(hr[hh], t)) {
            if (!k_waited) {
              if (!wait_all(bar(ctl->kv_full[kst]), kph)) { ok = false; break; }
              ptx::tc_fence_after();
              k_waited = true;
            }
            const uint64_t dq = dq0 + ((hh * Cfg::kTileBytes) >> 4);
            const uint64_t dk = dk0 + ((kst * Cfg::kTileBytes) >> 4);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
              const uint32_t off =
                  (ks / Cfg::kKStepsPerBlock) * Cfg::kBlockBytes + (ks % Cfg::kKStepsPerBlock) * 32;
              ptx::mma_ss_lead(lead, tmem + colS, dq + (off >> 4), dk + (off >> 4), Cfg::kIdescQK,
                               ks > 0 ? 1u : 0u);
            }
            ptx::mma_commit_lead(lead, bar(ctl->s_full[hh]));
            pend[hh] = true;
          }
        }
        if (!ok) break;
        if (!last) ptx::mma_commit_lead(lead, bar(ctl->kv_empty[kst]));       // K_t: free after its S MMAs
        if (i > 0) ptx::mma_commit_lead(lead, bar(ctl->kv_empty[prev_vst]));  // V_{t-1}: free after its P.V
        if (i == n_u - 1) ptx::mma_commit_lead(lead, bar(ctl->q_empty));      // Q: free after the last S MMA
        prev_vst = vst;
        prev_vph = vph;
      }
    }
    // Every MMA lane 0 issued has completed once `drain` flips.
    ptx::mma_commit_lead(lead, bar(ctl->drain));
    drain_wait(bar(ctl->drain), 0u);
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ SiLU + epilogue
    const int hh = warp >> 2;          // half
    const int quarter = warp & 3;      // TMEM lane quarter
    const int row = quarter * 32 + lane;  // row within the half
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t taddr_s = tmem + lane_off + (hh ? Cfg::kColS1 : Cfg::kColS0);
    const uint32_t taddr_o = tmem + lane_off + (hh ? Cfg::kColO1 : Cfg::kColO0);
    const float half_alpha = p.half_alpha;
    const float inv_n = p.inv_n;
    int slot = 0;
    uint32_t sched_full_par[2] = {0u, 0u};
    uint32_t s_full_par = 0u, o_full_par = 0u;
    bool ok = true;
    while (ok) {
      ok = wait_bounded(bar(ctl->sched_full[slot]), sched_full_par[slot], abort_flag, p.err, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      sched_full_par[slot] ^= 1u;
      const Work w = read_slot(ctl->slot[slot]);
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(ctl->sched_empty[slot]));
      slot ^= 1;
      if (!w.valid) break;

      const int lo = hh * kTileRows;
      const int nr = (w.nrows - lo) < kTileRows ? (w.nrows - lo) : kTileRows;
      if (nr <= 0) continue;
      const int p0 = w.pos0 + lo;
      const TileRange r = key_tiles(p0, p0 + nr, w.U);
      const int n = tile_count(r);
      const int i_pos = p0 + row;                      // this thread's query position
      const int lim_abs = (i_pos < w.U) ? i_pos + 1 : w.U;  // keys [0, lim_abs) visible, plus self
      const float* rab_row = kRab ? p.rab + (size_t)w.h * p.rab_len : nullptr;
      const int rab_max = kRab ? p.rab_len - 1 : 0;
      for (int k = 0; k < n; ++k) {
        const int j0 = tile_at(r, k) * kTileRows;
        ok = wait_bounded(bar(ctl->s_full[hh]), s_full_par, abort_flag, p.err, p.wait_limit_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        s_full_par ^= 1u;
        ptx::tc_fence_after();
        const bool full = (j0 + kTileRows <= w.U) && (j0 + kTileRows <= p0 + 1);
        const int lim = lim_abs - j0;
        const int self = i_pos - j0;
        const int rel0 = i_pos - j0;
        // 32-column chunks: the load of chunk c+1 is in flight while chunk c is computed.
        if constexpr (kRab) {
          // The bias reads need registers the next chunk's load would hold: one chunk at a time.
          uint32_t ra[32];
          ptx::tmem_ld32(taddr_s + 0, ra);
          ptx::tmem_ld_wait(ra);
          silu_chunk<0, kRab>(ra, taddr_s, half_alpha, full, lim, self, rab_row, rel0, rab_max);
          ptx::tmem_ld32(taddr_s + 32, ra);
          ptx::tmem_ld_wait(ra);
          silu_chunk<1, kRab>(ra, taddr_s, half_alpha, full, lim, self, rab_row, rel0, rab_max);
          ptx::tmem_ld32(taddr_s + 64, ra);
          ptx::tmem_ld_wait(ra);
          silu_chunk<2, kRab>(ra, taddr_s, half_alpha, full, lim, self, rab_row, rel0, rab_max);
          ptx::tmem_ld32(taddr_s + 96, ra);
          ptx::tmem_ld_wait(ra);
          silu_chunk<3, kRab>(ra, taddr_s, half_alpha, full, lim, self, rab_row, rel0, rab_max);
        } else {
          uint32_t ra[32], rb[32];
          ptx::tmem_ld32(taddr_s + 0, ra);
          ptx::tmem_ld_wait(ra);
          ptx::tmem_ld32(taddr_s + 32, rb);
          silu_chunk<0, kRab>(ra, taddr_s, half_alpha, full, lim, self, rab_row, rel0, rab_max);
          ptx::tmem_ld_wait(rb);
          ptx::tmem_ld32(taddr_s + 64, ra);
          silu_chunk<1, kRab>(rb, taddr_s, half_alpha, full, lim, self, rab_row, rel0, rab_max);
          ptx::tmem_ld_wait(ra);
          ptx::tmem_ld32(taddr_s + 96, rb);
          silu_chunk<2, kRab>(ra, taddr_s, half_alpha, full, lim, self, rab_row, rel0, rab_max);
          ptx::tmem_ld_wait(rb);
          silu_chunk<3, kRab>(rb, taddr_s, half_alpha, full, lim, self, rab_row, rel0, rab_max);
        }
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(ctl->p_full[hh]));
      }
      if (!ok) break;
      // Epilogue: O_h * (1/N) -> bf16 -> out rows that exist.
      ok = wait_bounded(bar(ctl->o_full[hh]), o_full_par, abort_flag, p.err, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      o_full_par ^= 1u;
      ptx::tc_fence_after();
      const size_t orow = (size_t)(w.q_row0 + lo + row);
      __nv_bfloat16* dst = p.out + orow * p.out_ld + (size_t)w.h * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ro[32];
        ptx::tmem_ld32(taddr_o + c * 32, ro);
        ptx::tmem_ld_wait(ro);
        if (row < nr) {
          uint4 a4[4];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            a4[q4].x = pack_bf16x2(__uint_as_float(ro[q4 * 8 + 0]) * inv_n, __uint_as_float(ro[q4 * 8 + 1]) * inv_n);
            a4[q4].y = pack_bf16x2(__uint_as_float(ro[q4 * 8 + 2]) * inv_n, __uint_as_float(ro[q4 * 8 + 3]) * inv_n);
            a4[q4].z = pack_bf16x2(__uint_as_float(ro[q4 * 8 + 4]) * inv_n, __uint_as_float(ro[q4 * 8 + 5]) * inv_n);
            a4[q4].w = pack_bf16x2(__uint_as_float(ro[q4 * 8 + 6]) * inv_n, __uint_as_float(ro[q4 * 8 + 7]) * inv_n);
            reinterpret_cast<uint4*>(dst + c * 32)[q4] = a4[q4];
          }
          if (p.gate != nullptr) {
            // Layer epilogue: the gate row U, a copy of it and U * A, beside A in the next
            // projection's input.
            const size_t col = (size_t)w.h * D + c * 32;
            const uint4* u4 = reinterpret_cast<const uint4*>(p.gate + orow * p.gate_ld + col);
            uint4* cp4 = reinterpret_cast<uint4*>(p.gate_copy + orow * p.out_ld + col);
            uint4* pr4 = reinterpret_cast<uint4*>(p.gate_prod + orow * p.out_ld + col);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const uint4 u = u4[q4];
              cp4[q4] = u;
              uint4 pr;
              pr.x = mul_bf16x2(u.x, a4[q4].x);
              pr.y = mul_bf16x2(u.y, a4[q4].y);
              pr.z = mul_bf16x2(u.z, a4[q4].z);
              pr.w = mul_bf16x2(u.w, a4[q4].w);
              pr4[q4] = pr;
            }
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(ctl->o_empty[hh]));
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == kMmaWarp) ptx::tmem_dealloc(tmem, Cfg::kTmemCols);
  // The last CTA to finish re-arms the plan's work counter, so the same plan can be replayed.
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.done_counter, 1) == (int)gridDim.x - 1) {
      atomicExch(p.work_counter, 0);
      atomicExch(p.done_counter, 0);
    }
  }
}

// Self-check of the failure path: one thread waits, through the bounded wait every role of the
// attention kernel uses, on an mbarrier that nothing ever arrives on.  After limit_ns the wait
// gives up, records kErrTimeout in the error word and raises the abort flag, and the kernel
// returns normally: no trap, no hang, and the context stays usable.
__global__ void wait_timeout_selfcheck_kernel(unsigned* err, uint64_t limit_ns) {
  __shared__ uint64_t never;
  __shared__ int32_t abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(ptx::smem_addr(&never), 1);
    abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) wait_bounded(ptx::smem_addr(&never), 0u, &abort_flag, err, limit_ns);
}

}  // namespace hstu
