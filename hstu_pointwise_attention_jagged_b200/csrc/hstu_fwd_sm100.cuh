// hstu_fwd_sm100.cuh — fused forward kernel of jagged target-aware HSTU pointwise attention for
// sm_100a:  out = Mask(SiLU(alpha * Q K^T)) V / N   (DLRMv3 review, section "model selection").
//
// One persistent CTA per SM pulls work items (user b, head h, one tile of up to 128 query rows)
// from a cost-ordered list through an atomic counter.  Every role walks the same global sequence
// of score tiles g = 0, 1, 2, ... over the CTA's query tiles and their visible key tiles.
//
//   warp 8       producer: fetches the next item, TMA-loads each query tile's Q into its buffer
//                (one of two at d <= 64) and the K and V tiles into a ring of shared-memory
//                slots, in the order the tensor core consumes them: K_0 K_1 K_2 V_0 K_3 V_1 K_4
//                ... (V_{g-3}, K_g).
//   warp 9       MMA issuer (lane 0 issues every tcgen05 instruction).  Group g is
//                O += P_{g-3} V_{g-3}  (TS form, P read from TMEM), then S_g = Q K_g^T into score
//                buffer g mod 3 (SS form), then one commit.  Three score buffers give the SiLU of
//                tile g two whole groups of tensor-core work to hide behind before P_g is needed.
//   warps 0-3,   SiLU warpgroups; warpgroup g mod 2 takes tile g: TMEM -> registers, p = mask ?
//   warps 4-7    silu(alpha*s) : 0 with silu(x) = h + h*tanh(h), h = x/2 (one MUFU op per score),
//                packed to bf16 and written back over S_g in TMEM.
//   warps 10-13  epilogue: after a query tile's last P.V, O * (1/N) -> bf16 -> row-predicated
//                global stores.  O is released as soon as it is in registers, so the next
//                query tile's first P.V waits only for the TMEM reads.
//
// TMEM (512 columns x 128 lanes of fp32): O [0, D), score buffer b at [128 + 128 b, 256 + 128 b)
// for b = 0, 1, 2.  P_g (bf16 pairs) overwrites the first 64 columns of its score buffer; the
// next S MMA into that buffer is issued after the P.V that reads it, and tcgen05 MMAs from one
// thread execute in order.
//
// Each group has one ready barrier: the producer's copies for it (Q with a query tile's first key tile,
// V_{g-3}, K_g) complete their bytes on it and the four SiLU warps that wrote P_{g-3} arrive on it,
// so the MMA warp makes one wait per group.  A ring slot is reused once the group that consumed
// its previous tile has completed; the score commit of group G covers every MMA issued before it,
// so the producer waits on that commit and no separate release commit is needed.
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

constexpr int kSCommits = 6;      // score-commit barriers: tile g's S commit arrives on s_full[g mod 6]
constexpr int kGroupBars = 8;     // group-ready barriers: group g waits on g_ready[g mod 8]

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
  // Q buffers and K/V ring slots in 227 KB.  At d = 128 one Q buffer and six slots: a K or V copy
  // from L2 takes longer than a group of MMAs, so the sixth slot, which lets the producer run a whole
  // group further ahead, is worth more than loading the next query tile's Q early.  At d <= 64 two
  // Q buffers and ten slots fit.
  static constexpr int kQBufs = (D == 128) ? 1 : 2;
  static constexpr int kStages = (D == 128) ? 6 : 10;
  static constexpr int kSBufs = 3;
  // The producer reuses a ring slot after waiting on the score commit of the group that consumed
  // the slot's previous tile.  That commit rotates over kSCommits barriers, so the wait is
  // unambiguous only while group G + kSCommits cannot have completed yet, i.e. while its K tile
  // (load 2 (G + kSCommits) - 2) is not yet loaded: at worst (G = 0, load kStages) that needs
  // kStages <= 2 kSCommits - 2.
  static_assert(kStages <= 2 * kSCommits - 2, "ring deeper than the score commits can track");
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 0, kColS = 128;  // score buffer b at kColS + 128 b
  static constexpr int kSmemTiles = (kQBufs + kStages) * kTileBytes;
  static constexpr int kSmemBytes = 1024 + kSmemTiles + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory");
  static constexpr uint32_t kIdescQK = ptx::idesc_bf16_f32(128, 128, false);
  static constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(128, D, true);
};

constexpr int kNumThreads = 448;  // 8 SiLU warps + producer + MMA issuer + 4 epilogue warps
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;       // issues every MMA and owns the TMEM allocation
constexpr int kEpiWarp0 = 10;     // first of the four epilogue warps
constexpr int kSlots = 4;         // work-item slots between the producer and the other roles
constexpr uint64_t kWaitLimitNs = 4000000000ull;  // 4 s per wait
constexpr uint64_t kDrainLimitNs = 200000000ull;  // 0.2 s per drain wait on the abort path
constexpr uint64_t kCopyGraceNs = 1000000ull;     // 1 ms for the copies in flight on the abort path

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
  uint64_t q_empty[2];
  uint64_t g_ready[kGroupBars];  // group g: its Q/V/K bytes and P_{g-3} are in
  uint64_t s_full[kSCommits];
  uint64_t o_full, o_empty;
  uint64_t sched_full[kSlots], sched_empty[kSlots];
  uint64_t drain;
  // work slot: valid, h, kv_start, q_row0, pos0, nrows, L, U
  int32_t slot[kSlots][8];
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

// Limits below this are test limits: their waits poll instead of suspending in try_wait, whose
// suspension may last until the phase completes, so that the clock is read every few clocks.
constexpr uint64_t kPollBelowNs = 1000000ull;

__device__ __forceinline__ uint32_t suspend_hint(uint64_t limit_ns) {
  return limit_ns < 0xffffffffull ? (uint32_t)limit_ns : 0xffffffffu;
}

// Slow path of wait_bounded: waits until the phase completes, the CTA aborts, or the time limit.
// Each try_wait may itself suspend the thread for a while, so the flag and the clock are checked
// after every attempt.
__device__ __noinline__ bool wait_bounded_slow(uint32_t bar, uint32_t parity, volatile int32_t* abort_flag,
                                               unsigned* err, uint64_t limit_ns) {
  const uint64_t t0 = ptx::globaltimer_ns();
  const bool poll = limit_ns < kPollBelowNs;
  while (true) {
    if (poll ? ptx::mbar_test_wait(bar, parity) : ptx::mbar_try_wait_for(bar, parity, suspend_hint(limit_ns)))
      return true;
    if (*abort_flag) return false;
    if (ptx::globaltimer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicOr(err, kErrTimeout);
      return false;
    }
  }
}

// Waits for phase `parity` of `bar`; false if the CTA is aborting or this wait timed out.  The
// first try is inline (a call right after a burst of MMAs stalls the issuing warp) and may
// suspend the thread until the phase completes; a wait with a test limit goes straight to the
// polling slow path instead.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int32_t* abort_flag,
                                             unsigned* err, uint64_t limit_ns = kWaitLimitNs) {
  if (limit_ns >= kPollBelowNs && ptx::mbar_try_wait_for(bar, parity, 0xffffffffu)) return true;
  return wait_bounded_slow(bar, parity, abort_flag, err, limit_ns);
}

// Abort-path drain: waits for phase `parity` of `bar` for at most kDrainLimitNs.
__device__ __noinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = ptx::globaltimer_ns();
  while (!ptx::mbar_try_wait_for(bar, parity, (uint32_t)kDrainLimitNs))
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
// With kRab, a visible pair also gets bias[c] (load_bias: rab_row[min(rel0 - c, rab_max)], its
// query-key distance clipped to the last table entry; rel0 = query position - first key of the
// tile).
// The 32 biases of chunk kChunk of this row: column c has distance rel0 - 32*kChunk - c, clipped
// to [0, rab_max] (negative distances are masked pairs).  The loads are issued together, ahead of
// the chunk's TMEM load, so their latency is paid once per chunk rather than once per pair.  A
// warp's load of one column reads 32 consecutive entries (the rows' distances differ by one).
template <int kChunk>
__device__ __forceinline__ void load_bias(float (&b)[32], const float* rab_row, int rel0, int rab_max) {
  const int hi = rel0 - kChunk * 32;
  if (hi >= 31 && hi <= rab_max) {
#pragma unroll
    for (int c = 0; c < 32; ++c) b[c] = __ldg(rab_row + hi - c);
  } else {
#pragma unroll
    for (int c = 0; c < 32; ++c) b[c] = __ldg(rab_row + min(max(hi - c, 0), rab_max));
  }
}

template <int kChunk, bool kRab, bool kMasked>
__device__ __forceinline__ void silu_chunk(const uint32_t (&r)[32], uint32_t taddr_s, float half_alpha,
                                           int lim, int self, const float (&bias)[32]) {
  uint32_t pk[16];
  // Columns are taken in pairs on the two-wide FMA pipe: h = s * alpha/2 and p = h * tanh(h) + h,
  // bit-identical to the scalar forms.
  const uint64_t ha2 = ptx::f32x2(half_alpha, half_alpha);
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const uint64_t h2 = ptx::mul_f32x2(ptx::f32x2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1])), ha2);
    float h0, h1;
    ptx::f32x2_split(h2, h0, h1);
    float p0, p1;
    ptx::f32x2_split(ptx::fma_f32x2(h2, ptx::f32x2(ptx::tanh_approx(h0), ptx::tanh_approx(h1)), h2), p0, p1);
    if constexpr (kRab) {
      p0 += bias[2 * e];
      p1 += bias[2 * e + 1];
    }
    if constexpr (kMasked) {
      const int c0 = kChunk * 32 + 2 * e;
      p0 = (c0 < lim || c0 == self) ? p0 : 0.0f;
      p1 = (c0 + 1 < lim || c0 + 1 == self) ? p1 : 0.0f;
    }
    pk[e] = pack_bf16x2(p0, p1);
  }
  ptx::tmem_st16(taddr_s + kChunk * 16, pk);
}

// The SiLU of one score tile for this thread's row: four 32-column chunks, each read from TMEM,
// transformed and written back as packed bf16 over the first 64 columns.  A tile that lies inside
// every one of its rows' visible ranges takes the kMasked = false form, which has no per-column
// tests at all; only tiles that cross the diagonal or the history edge take the masked form.
// Chunks are loaded one at a time: the registers a second buffer would take keep the SiLU free of
// spills, and the other SiLU warps on the scheduler cover the load latency.  With kRab, the next
// chunk's biases are loaded as soon as the previous chunk is done.
template <bool kMasked, bool kRab>
__device__ __forceinline__ void silu_tile(uint32_t taddr_s, float half_alpha, int lim, int self, float (&bias)[32],
                                          const float* rab_row, int rel0, int rab_max) {
  uint32_t ra[32];
  ptx::tmem_ld32(taddr_s + 0, ra);
  ptx::tmem_ld_wait(ra);
  silu_chunk<0, kRab, kMasked>(ra, taddr_s, half_alpha, lim, self, bias);
  if constexpr (kRab) load_bias<1>(bias, rab_row, rel0, rab_max);
  ptx::tmem_ld32(taddr_s + 32, ra);
  ptx::tmem_ld_wait(ra);
  silu_chunk<1, kRab, kMasked>(ra, taddr_s, half_alpha, lim, self, bias);
  if constexpr (kRab) load_bias<2>(bias, rab_row, rel0, rab_max);
  ptx::tmem_ld32(taddr_s + 64, ra);
  ptx::tmem_ld_wait(ra);
  silu_chunk<2, kRab, kMasked>(ra, taddr_s, half_alpha, lim, self, bias);
  if constexpr (kRab) load_bias<3>(bias, rab_row, rel0, rab_max);
  ptx::tmem_ld32(taddr_s + 96, ra);
  ptx::tmem_ld_wait(ra);
  silu_chunk<3, kRab, kMasked>(ra, taddr_s, half_alpha, lim, self, bias);
}

// Loads run K_0 K_1 K_2 | V_0 K_3 | V_1 K_4 | ... in the order the MMA warp consumes them, so load
// e < 3 is consumed by group e and load e >= 3 by group (e + 3) / 2.  (The closing one to three V
// loads of the CTA, consumed by P.V-only groups, are never looked up: no load follows them by a
// whole ring.)
__device__ __forceinline__ int group_of_load(int e) { return e < 3 ? e : (e + 3) >> 1; }

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
  const uint32_t sQ = sbase;                                   // kQBufs tiles
  const uint32_t sKV = sbase + Cfg::kQBufs * Cfg::kTileBytes;  // kStages tiles
  auto* ctl = reinterpret_cast<SmemCtl<Cfg::kStages>*>(smem + Cfg::kSmemTiles);
  volatile int32_t* abort_flag = &ctl->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  auto bar = [](const uint64_t& b) { return ptx::smem_addr(&b); };

  if (warp == kProducerWarp && lane == 0) {
    for (int i = 0; i < 2; ++i) ptx::mbar_init(bar(ctl->q_empty[i]), 1);
    // The producer's expect-tx arrival plus one arrival per warp of the SiLU warpgroup.
    for (int i = 0; i < kGroupBars; ++i) ptx::mbar_init(bar(ctl->g_ready[i]), 1 + 4);
    for (int b = 0; b < kSCommits; ++b) ptx::mbar_init(bar(ctl->s_full[b]), 1);
    ptx::mbar_init(bar(ctl->o_full), 1);
    ptx::mbar_init(bar(ctl->o_empty), 4);      // one arrival per epilogue warp
    for (int s = 0; s < kSlots; ++s) {
      ptx::mbar_init(bar(ctl->sched_full[s]), 1);
      ptx::mbar_init(bar(ctl->sched_empty[s]), 1 + 8 + 4);  // MMA, SiLU and epilogue warps
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
      uint32_t sched_empty_par = (1u << kSlots) - 1u;  // bit s: parity of slot s's next wait
      int sub = 0;        // query tiles whose Q load was issued
      int j = 0;          // K/V loads issued
      int g = 0;          // score tiles (groups with an S) armed
      int armed_hi = 0;   // one past the highest group index armed
      bool q_unarmed = false;  // a Q copy is on group g's barrier, whose arrival is still to come
      // V rows and heads of tiles g-3, g-2, g-1.
      int vrow0 = 0, vrow1 = 0, vrow2 = 0, vh0 = 0, vh1 = 0, vh2 = 0;
      bool ok = true;
      // True once ring slot e mod kStages is free: the group that consumed the slot's previous
      // tile (load e - kStages) has completed.
      auto slot_free = [&](int e) {
        if (e < Cfg::kStages) return true;
        const int G = group_of_load(e - Cfg::kStages);
        return wait_bounded(bar(ctl->s_full[G % kSCommits]), (uint32_t)((G / kSCommits) & 1), abort_flag, p.err,
                            p.wait_limit_ns);
      };
      auto tma_tile = [&](const CUtensorMap* tm, uint32_t dst, uint32_t rb, int col0, int row) {
        for (int blk = 0; blk < Cfg::kBlocks; ++blk)
          ptx::tma_load_2d(dst + blk * Cfg::kBlockBytes, tm, rb, col0 + blk * Cfg::kBlockElems, row);
      };
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
          w.q_row0 = p.q_start[b] + pair * kItemRows;
          w.pos0 = c + pair * kItemRows;
          const int rows = (w.L - c) - pair * kItemRows;
          w.nrows = rows < kItemRows ? rows : kItemRows;
        }
        if (!wait_bounded(bar(ctl->sched_empty[slot]), (sched_empty_par >> slot) & 1u, abort_flag, p.err,
                          p.wait_limit_ns)) {
          ok = false;
          break;
        }
        sched_empty_par ^= 1u << slot;
        volatile int32_t* s = ctl->slot[slot];
        s[0] = w.valid; s[1] = w.h; s[2] = w.kv_start; s[3] = w.q_row0;
        s[4] = w.pos0; s[5] = w.nrows; s[6] = w.L; s[7] = w.U;
        ptx::mbar_arrive(bar(ctl->sched_full[slot]));
        slot = (slot + 1) & (kSlots - 1);
        if (!w.valid) break;

        {
          const TileRange r = key_tiles(w.pos0, w.pos0 + w.nrows, w.U);
          const int n = tile_count(r);
          const int qb = sub % Cfg::kQBufs;
          if (!wait_bounded(bar(ctl->q_empty[qb]), (uint32_t)(((sub / Cfg::kQBufs) & 1) ^ 1), abort_flag, p.err,
                            p.wait_limit_ns)) {
            ok = false;
            break;
          }
          // The query tile's Q goes out at once, ahead of its first K and V tiles, which wait for
          // ring slots: its bytes join the first group's barrier without an arrival, and the
          // producer's one arrival for that group comes with the K/V bytes below.  (Group g - 8's
          // phase on that barrier completed before group g - 1 was armed.)
          {
            const uint32_t rb = bar(ctl->g_ready[g & (kGroupBars - 1)]);
            ptx::mbar_expect_tx(rb, Cfg::kTileBytes);
            tma_tile(&tm_q, sQ + qb * Cfg::kTileBytes, rb, w.h * D, w.q_row0);
            ++sub;
            q_unarmed = true;
          }
          for (int k = 0; k < n; ++k) {
            // Group g reads V_{g-3} (load j) and K_g (load j+1), or K_g alone for g < 3; they and
            // (on a query tile's first tile) Q land on the group's ready barrier.
            const bool has_v = g >= 3;
            if (!slot_free(j) || (has_v && !slot_free(j + 1))) { ok = false; break; }
            const int krow = w.kv_start + tile_at(r, k) * kTileRows;
            const uint32_t rb = bar(ctl->g_ready[g & (kGroupBars - 1)]);
            ptx::mbar_arrive_expect_tx(rb, Cfg::kTileBytes * (1 + (has_v ? 1 : 0)));
            if (!has_v)  // no P.V in this group: stand in for the SiLU warps' arrivals
              for (int a = 0; a < 4; ++a) ptx::mbar_arrive(rb);
            q_unarmed = false;
            if (has_v) {
              tma_tile(&tm_v, sKV + (j % Cfg::kStages) * Cfg::kTileBytes, rb, vh0 * D, vrow0);
              ++j;
            }
            tma_tile(&tm_k, sKV + (j % Cfg::kStages) * Cfg::kTileBytes, rb, w.h * D, krow);
            ++j;
            vrow0 = vrow1; vh0 = vh1;
            vrow1 = vrow2; vh1 = vh2;
            vrow2 = krow;  vh2 = w.h;
            armed_hi = ++g;
          }
        }
      }
      // The closing groups t + 3 carry the V tiles of the last (up to) three score tiles t.
      for (int t = (g >= 3 ? g - 3 : 0); t < g && ok; ++t) {
        const int i = t - g + 3;  // 0, 1, 2 <-> tiles g-3, g-2, g-1
        const int row = i == 0 ? vrow0 : (i == 1 ? vrow1 : vrow2);
        const int h = i == 0 ? vh0 : (i == 1 ? vh1 : vh2);
        if (!slot_free(j)) { ok = false; break; }
        const uint32_t rb = bar(ctl->g_ready[(t + 3) & (kGroupBars - 1)]);
        ptx::mbar_arrive_expect_tx(rb, Cfg::kTileBytes);
        tma_tile(&tm_v, sKV + (j % Cfg::kStages) * Cfg::kTileBytes, rb, h * D, row);
        ++j;
        armed_hi = t + 4;
      }
      if (*abort_flag) {
        // Let every copy this CTA started land before its shared memory is released.  A group
        // barrier's phase completes once its bytes and the SiLU warps' arrivals are in, and the
        // arrivals of an aborted group may never come.  Arriving for them here is not an option:
        // if they did come while bytes were still outstanding, the extra arrival would land on a
        // phase with no arrivals pending, which is not defined.  So the producer only waits, on
        // each barrier still in use, all within one budget of kCopyGraceNs: every phase complete
        // means every copy landed, and otherwise the whole budget, a thousand times a copy's
        // duration, has passed.
        const uint64_t t0 = ptx::globaltimer_ns();
        for (int x = armed_hi > kGroupBars ? armed_hi - kGroupBars : 0; x < armed_hi; ++x) {
          if (x >= g && x < 3) continue;  // group indices never used when the CTA had < 3 tiles
          const uint32_t rb = bar(ctl->g_ready[x & (kGroupBars - 1)]);
          const uint32_t par = (uint32_t)((x / kGroupBars) & 1);
          while (!ptx::mbar_test_wait(rb, par) && ptx::globaltimer_ns() - t0 < kCopyGraceNs) {
          }
        }
        // A Q copy on a group that was never armed: that phase cannot complete, so the budget runs.
        while (q_unarmed && ptx::globaltimer_ns() - t0 < kCopyGraceNs) {
        }
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop in step, so the control flow is uniform and the descriptors
    // and TMEM addresses stay in uniform registers; lane 0 alone issues the tcgen05 instructions
    // (the *_lead forms), so every MMA and commit comes from one thread, as commit tracking needs.
    // The loop keeps its ring slot, buffer and barrier indices as running counters: every
    // instruction between two MMA bursts is tensor-core idle time.
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
    uint32_t sched_full_par = 0u;  // bit s: parity of slot s's next wait
    int sub = 0;
    int g = 0;               // groups with an S issued
    int st = 0;              // ring slot of the next tile to consume
    uint32_t b3 = 0;         // g mod 3: score buffer of S_g, and of P_{g-3}
    int c6 = 0;              // g mod kSCommits: barrier of S_g's commit
    int r8 = 0;              // g mod kGroupBars: ready barrier of group g
    uint32_t rpar = 0u;      // parity of that barrier's phase for group g
    uint32_t o_empty_par = 1u;
    // Tiles g-3, g-2, g-1: bit 0 = first tile of its query tile, bit 1 = last tile of its query tile.
    uint32_t f0 = 0, f1 = 0, f2 = 0;
    bool ok = true;
    // O += P V for a tile whose P is in score buffer pb and whose V is in ring slot vs (its group's
    // ready barrier already waited).  A query tile's first tile starts O afresh once the epilogue
    // has read the previous O; its last one commits O to the epilogue.
    auto issue_pv = [&](uint32_t pb, int vs, uint32_t flags) {
      if (flags & 1u) {
        if (!wait_all(bar(ctl->o_empty), o_empty_par)) return false;
        o_empty_par ^= 1u;
      }
      ptx::tc_fence_after();
      const uint64_t dv = dv0 + ((vs * Cfg::kTileBytes) >> 4);
      const uint32_t colP = Cfg::kColS + 128u * pb;
#pragma unroll
      for (int ks = 0; ks < kTileRows / 16; ++ks)
        ptx::mma_ts_lead(lead, tmem + Cfg::kColO, tmem + colP + ks * 8, dv + ((ks * 16 * Cfg::kRowBytes) >> 4),
                         Cfg::kIdescPV, ((flags & 1u) && ks == 0) ? 0u : 1u);
      if (flags & 2u) ptx::mma_commit_lead(lead, bar(ctl->o_full));
      return true;
    };
    auto next_slot = [](int s) { return s + 1 == Cfg::kStages ? 0 : s + 1; };
    while (ok) {
      if (!wait_all(bar(ctl->sched_full[slot]), (sched_full_par >> slot) & 1u)) {
        ok = false;
        break;
      }
      sched_full_par ^= 1u << slot;
      const Work w = read_slot(ctl->slot[slot]);
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(ctl->sched_empty[slot]));
      slot = (slot + 1) & (kSlots - 1);
      if (!w.valid) break;

      {
        const TileRange r = key_tiles(w.pos0, w.pos0 + w.nrows, w.U);
        const int n = tile_count(r);
        const int qb = sub % Cfg::kQBufs;
        const uint64_t dq = dq0 + ((qb * Cfg::kTileBytes) >> 4);
        for (int k = 0; k < n; ++k) {
          // Group g: once its tiles and P_{g-3} are in, the P.V of tile g-3, then the scores of
          // tile g into buffer g mod 3, then one commit.
          if (!wait_all(bar(ctl->g_ready[r8]), rpar)) { ok = false; break; }
          ptx::tc_fence_after();
          if (g >= 3) {
            if (!issue_pv(b3, st, f0)) { ok = false; break; }
            st = next_slot(st);
          }
          const uint64_t dk = dk0 + ((st * Cfg::kTileBytes) >> 4);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t off =
                (ks / Cfg::kKStepsPerBlock) * Cfg::kBlockBytes + (ks % Cfg::kKStepsPerBlock) * 32;
            ptx::mma_ss_lead(lead, tmem + Cfg::kColS + 128u * b3, dq + (off >> 4), dk + (off >> 4), Cfg::kIdescQK,
                             ks > 0 ? 1u : 0u);
          }
          st = next_slot(st);
          ptx::mma_commit_lead(lead, bar(ctl->s_full[c6]));
          if (k == n - 1) ptx::mma_commit_lead(lead, bar(ctl->q_empty[qb]));  // Q: free after its last S
          f0 = f1;
          f1 = f2;
          f2 = (k == 0 ? 1u : 0u) | (k == n - 1 ? 2u : 0u);
          ++g;
          b3 = (b3 == 2u) ? 0u : b3 + 1u;
          c6 = (c6 == kSCommits - 1) ? 0 : c6 + 1;
          r8 = (r8 + 1) & (kGroupBars - 1);
          if (r8 == 0) rpar ^= 1u;
        }
        ++sub;
      }
    }
    // The closing groups t + 3: the P.V of the last (up to) three tiles t.
    for (int t = (g >= 3 ? g - 3 : 0); t < g && ok; ++t) {
      const int i = t - g + 3;  // 0, 1, 2 <-> tiles g-3, g-2, g-1
      const int x = t + 3;
      ok = wait_all(bar(ctl->g_ready[x & (kGroupBars - 1)]), (uint32_t)((x / kGroupBars) & 1)) &&
           issue_pv((uint32_t)(t % 3), st, i == 0 ? f0 : (i == 1 ? f1 : f2));
      st = next_slot(st);
    }
    // Every MMA lane 0 issued has completed once `drain` flips.
    ptx::mma_commit_lead(lead, bar(ctl->drain));
    drain_wait(bar(ctl->drain), 0u);
    __syncwarp();
  } else if (warp < kProducerWarp) {
    // ------------------------------------------------------------------ SiLU
    const int wg = warp >> 2;          // takes the score tiles g with g mod 2 == wg
    const int quarter = warp & 3;      // TMEM lane quarter
    const int row = quarter * 32 + lane;  // row within the query tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float half_alpha = p.half_alpha;
    int slot = 0;
    uint32_t sched_full_par = 0u;
    int g = 0;
    bool ok = true;
    while (ok) {
      ok = wait_bounded(bar(ctl->sched_full[slot]), (sched_full_par >> slot) & 1u, abort_flag, p.err,
                        p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      sched_full_par ^= 1u << slot;
      const Work w = read_slot(ctl->slot[slot]);
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(ctl->sched_empty[slot]));
      slot = (slot + 1) & (kSlots - 1);
      if (!w.valid) break;

      const float* rab_row = kRab ? p.rab + (size_t)w.h * p.rab_len : nullptr;
      const int rab_max = kRab ? p.rab_len - 1 : 0;
      {
        const int p0 = w.pos0;
        const TileRange r = key_tiles(p0, p0 + w.nrows, w.U);
        const int n = tile_count(r);
        const int i_pos = p0 + row;                           // this thread's query position
        const int lim_abs = (i_pos < w.U) ? i_pos + 1 : w.U;  // keys [0, lim_abs) visible, plus self
        for (int k = (g + wg) & 1; k < n; k += 2) {
          const int gt = g + k;
          const int b = gt % 3;
          const uint32_t taddr_s = tmem + lane_off + Cfg::kColS + 128u * b;
          // The first chunk's biases do not depend on S: load them while S is computed.
          const int j0 = tile_at(r, k) * kTileRows;
          float bias[32];
          if constexpr (kRab) load_bias<0>(bias, rab_row, i_pos - j0, rab_max);
          ok = wait_bounded(bar(ctl->s_full[gt % kSCommits]), (uint32_t)((gt / kSCommits) & 1), abort_flag, p.err,
                            p.wait_limit_ns);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          ptx::tc_fence_after();
          const bool full = (j0 + kTileRows <= w.U) && (j0 + kTileRows <= p0 + 1);
          const int lim = lim_abs - j0;
          const int self = i_pos - j0;
          const int rel0 = i_pos - j0;
          // `full` is the same for every row of the tile, so the warp takes one branch.
          if (full) {
            silu_tile<false, kRab>(taddr_s, half_alpha, lim, self, bias, rab_row, rel0, rab_max);
          } else {
            silu_tile<true, kRab>(taddr_s, half_alpha, lim, self, bias, rab_row, rel0, rab_max);
          }
          ptx::tmem_st_wait();
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(bar(ctl->g_ready[(gt + 3) & (kGroupBars - 1)]));  // P_gt, for group gt+3
        }
        g += n;
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int quarter = warp & 3;         // TMEM lane quarter
    const int row = quarter * 32 + lane;  // row within the query tile
    const uint32_t taddr_o = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + Cfg::kColO;
    const float inv_n = p.inv_n;
    int slot = 0;
    uint32_t sched_full_par = 0u, o_full_par = 0u;
    bool ok = true;
    while (ok) {
      ok = wait_bounded(bar(ctl->sched_full[slot]), (sched_full_par >> slot) & 1u, abort_flag, p.err,
                        p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      sched_full_par ^= 1u << slot;
      const Work w = read_slot(ctl->slot[slot]);
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(ctl->sched_empty[slot]));
      slot = (slot + 1) & (kSlots - 1);
      if (!w.valid) break;

      {
        const int nr = w.nrows;
        ok = wait_bounded(bar(ctl->o_full), o_full_par, abort_flag, p.err, p.wait_limit_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        o_full_par ^= 1u;
        ptx::tc_fence_after();
        // O * (1/N) -> bf16 pairs in registers; O is then released to the next query tile's P.V.
        uint32_t a[D / 2];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ro[32];
          ptx::tmem_ld32(taddr_o + c * 32, ro);
          ptx::tmem_ld_wait(ro);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            a[c * 16 + e] = pack_bf16x2(__uint_as_float(ro[2 * e]) * inv_n, __uint_as_float(ro[2 * e + 1]) * inv_n);
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(ctl->o_empty));
        if (row < nr) {
          const size_t orow = (size_t)(w.q_row0 + row);
          const size_t col = (size_t)w.h * D;
          uint4* dst = reinterpret_cast<uint4*>(p.out + orow * p.out_ld + col);
#pragma unroll
          for (int q4 = 0; q4 < D / 8; ++q4)
            dst[q4] = make_uint4(a[4 * q4], a[4 * q4 + 1], a[4 * q4 + 2], a[4 * q4 + 3]);
          if (p.gate != nullptr) {
            // Layer epilogue: the gate row U, a copy of it and U * A, beside A in the next
            // projection's input.
            const uint4* u4 = reinterpret_cast<const uint4*>(p.gate + orow * p.gate_ld + col);
            uint4* cp4 = reinterpret_cast<uint4*>(p.gate_copy + orow * p.out_ld + col);
            uint4* pr4 = reinterpret_cast<uint4*>(p.gate_prod + orow * p.out_ld + col);
#pragma unroll
            for (int q4 = 0; q4 < D / 8; ++q4) {
              const uint4 u = u4[q4];
              cp4[q4] = u;
              uint4 pr;
              pr.x = mul_bf16x2(u.x, a[4 * q4]);
              pr.y = mul_bf16x2(u.y, a[4 * q4 + 1]);
              pr.z = mul_bf16x2(u.z, a[4 * q4 + 2]);
              pr.w = mul_bf16x2(u.w, a[4 * q4 + 3]);
              pr4[q4] = pr;
            }
          }
        }
      }
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
