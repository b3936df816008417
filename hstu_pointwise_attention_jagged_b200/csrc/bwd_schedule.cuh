// bwd_schedule.cuh — device-side work lists of the backward pass.
//
// The backward pass of out = Mask(SiLU(alpha Q K^T)) V / N (DLRMv3 review, section "model
// selection") runs as two persistent kernels over 128-row tiles of each user's segment:
//   - the dK/dV kernel owns one key tile and streams the query tiles that see it:
//       a history key tile (first key < U) is seen by every query tile from its own to the last
//       (history queries at or after it, and every candidate); a candidate-only key tile is seen
//       by its own query tile alone (a candidate sees itself among candidates);
//   - the dQ kernel owns one query tile and streams its visible key tiles, the same runs as the
//       forward pass.
// Both lists are sorted by cost (streamed tiles per item), largest first, so the persistent
// kernels run longest-processing-time-first.
#pragma once

#include <cstdint>

#include "schedule.cuh"

namespace hstu {

// Query tiles that see key tile kt of a segment of L tokens with U history tokens, as a
// TileRange ([0, e1) is always empty here).
__host__ __device__ __forceinline__ TileRange query_tiles_of_key_tile(int kt, int L, int U) {
  TileRange r{0, kt, kt + 1};
  if (kt * kTileRows < U) r.e2 = cdiv(L, kTileRows);
  return r;
}

// Key tiles visible to query tile qt (the forward pass's runs).
__host__ __device__ __forceinline__ TileRange key_tiles_of_query_tile(int qt, int L, int U) {
  const int p0 = qt * kTileRows;
  const int p1 = (p0 + kTileRows < L) ? p0 + kTileRows : L;
  return key_tiles(p0, p1, U);
}

// dS tiles of one head of a segment, kept for the dQ pass: one 128 x 128 tile per visible (key
// tile, query tile) pair, in key-tile order.  A history key tile kt pairs with query tiles
// kt .. T-1, a candidate-only key tile with its own query tile, so tile (kt, qt) sits at
// ds_tiles_before(kt) + (qt - kt).
__host__ __device__ __forceinline__ long long ds_tiles_before(int kt, int L, int U) {
  const long long T = cdiv(L, kTileRows), Th = cdiv(U, kTileRows), k = kt;
  if (k <= Th) return k * T - k * (k - 1) / 2;
  return Th * T - Th * (Th - 1) / 2 + (k - Th);
}
__host__ __device__ __forceinline__ long long ds_tiles_per_head(int L, int U) {
  return ds_tiles_before(cdiv(L, kTileRows), L, U);
}

struct BwdSchedArgs {
  const int32_t* seq_offsets;  // [B+1]
  const int32_t* num_targets;  // [B] or null
  int32_t B, H, total, max_seq_len, nbins, max_items;
  // Waves of users by first row (wave = row / wave_rows, at most nwaves - 1): items go by wave,
  // then by non-increasing cost, so the tiles streamed at one time stay in L2.
  int32_t wave_rows, nwaves;
  int32_t* header;      // [8] out: {dq counter, dq items, dq done, 0, kv counter, kv items, kv done, 0}
  int32_t* tile_start;  // [B+1] out: index of each user's first 128-row tile among all tiles
  long long* ds_base;   // [B+1] out: index of each user's first dS tile (all heads); may be null
  int4* dq_items;       // [max_items] out: {b, query tile, h, cost}, non-increasing cost
  int4* kv_items;       // [max_items] out: {b, key tile, h, cost}, non-increasing cost
  unsigned* err;
};

// One CTA of kSchedThreads threads: validates every user (a bad user sets kErrBadOffsets and gets
// no items), then writes both lists with a counting sort over (wave, cost) keys.
__global__ void __launch_bounds__(kSchedThreads) bwd_schedule_kernel(const BwdSchedArgs a) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ int hist[2][kMaxCostBins];
  __shared__ long long scan_scratch[2][32];
  __shared__ long long carry, carry_ds;
  __shared__ int s_L[kCachedUsers], s_U[kCachedUsers], s_ts[kCachedUsers + 1], s_w[kCachedUsers];
  const bool cached = a.B <= kCachedUsers;
  const int tid = threadIdx.x;
  const int nbins = a.nbins;
  const int nkeys = nbins * a.nwaves;  // <= kMaxCostBins (host)
  if (tid == 0) carry = carry_ds = 0;
  __syncthreads();

  // Pass 1: validation and tile starts.
  for (int base = 0; base < a.B; base += kSchedThreads) {
    const int b = base + tid;
    long long nt = 0, nds = 0;
    int L = 0, U = 0;
    if (b < a.B) {
      const int o0 = a.seq_offsets[b], o1 = a.seq_offsets[b + 1];
      const long long L64 = (long long)o1 - o0;
      const int T = a.num_targets ? a.num_targets[b] : 0;
      bool ok = o0 >= 0 && L64 >= 0 && o1 <= a.total && L64 <= a.max_seq_len && T >= 0 && T <= L64;
      if (b == 0 && o0 != 0) ok = false;
      if (b == a.B - 1 && o1 != a.total) ok = false;
      if (!ok) atomicOr(a.err, kErrBadOffsets);
      L = ok ? (int)L64 : 0;
      U = L - (ok ? T : 0);
      nt = cdiv(L, kTileRows);
      nds = ds_tiles_per_head(L, U);
    }
    long long incl = nt, incl_ds = nds, tot, tot_ds;
    block_inclusive_scan2(incl, incl_ds, scan_scratch, tot, tot_ds);
    const long long start = carry + incl - nt;
    if (b < a.B) {
      a.tile_start[b] = (int)start;
      if (a.ds_base) a.ds_base[b] = (carry_ds + incl_ds - nds) * a.H;
      if (cached) {
        s_L[b] = L;
        s_U[b] = U;
        s_ts[b] = (int)start;
        s_w[b] = min(a.seq_offsets[b] / a.wave_rows, a.nwaves - 1);
      }
    }
    __syncthreads();
    if (tid == 0) {
      carry += tot;
      carry_ds += tot_ds;
    }
    __syncthreads();
  }
  const int ntiles = (int)carry;
  if (tid == 0) {
    a.tile_start[a.B] = ntiles;
    if (a.ds_base) a.ds_base[a.B] = carry_ds * a.H;
    if (cached) s_ts[a.B] = ntiles;
  }
  __syncthreads();

  // Tile g: its user, its index within the user, and the user's L and U.  Users skipped in
  // pass 1 own no tiles.
  auto tile_of = [&](int g, int& b, int& t, int& L, int& U, int& wave) {
    b = owner_of(cached ? s_ts : a.tile_start, a.B, g);
    t = g - (cached ? s_ts[b] : a.tile_start[b]);
    if (cached) {
      L = s_L[b];
      U = s_U[b];
      wave = s_w[b];
    } else {
      L = a.seq_offsets[b + 1] - a.seq_offsets[b];
      U = L - (a.num_targets ? a.num_targets[b] : 0);
      wave = min(a.seq_offsets[b] / a.wave_rows, a.nwaves - 1);
    }
  };
  auto key_of = [&](int wave, int c) { return wave * nbins + (nbins - 1 - (c < nbins ? c : nbins - 1)); };

  // Both lists in one sweep: cost histograms, one two-value scan over the bins (costlier bins
  // first), then one scatter pass.  List 0 is the dQ list (items own a query tile), list 1 the
  // dK/dV list (items own a key tile).
  for (int i = tid; i < nkeys; i += kSchedThreads) {
    hist[0][i] = 0;
    hist[1][i] = 0;
  }
  __syncthreads();
  for (int g = tid; g < ntiles; g += kSchedThreads) {
    int b, t, L, U, wave;
    tile_of(g, b, t, L, U, wave);
    const int c0 = tile_count(key_tiles_of_query_tile(t, L, U));
    const int c1 = tile_count(query_tiles_of_key_tile(t, L, U));
    atomicAdd(&hist[0][key_of(wave, c0)], a.H);
    atomicAdd(&hist[1][key_of(wave, c1)], a.H);
  }
  __syncthreads();
  const int per = cdiv(nkeys, kSchedThreads);
  long long part0 = 0, part1 = 0;
  for (int k = 0; k < per; ++k) {
    const int key = tid * per + k;
    if (key < nkeys) {
      part0 += hist[0][key];
      part1 += hist[1][key];
    }
  }
  long long incl0 = part0, incl1 = part1, tot0, tot1;
  block_inclusive_scan2(incl0, incl1, scan_scratch, tot0, tot1);
  long long run0 = incl0 - part0, run1 = incl1 - part1;
  for (int k = 0; k < per; ++k) {
    const int key = tid * per + k;
    if (key < nkeys) {
      const int n0 = hist[0][key], n1 = hist[1][key];
      hist[0][key] = (int)run0;
      hist[1][key] = (int)run1;
      run0 += n0;
      run1 += n1;
    }
  }
  __syncthreads();
  if (tid < 2) {
    const long long tot = tid == 0 ? tot0 : tot1;
    a.header[4 * tid + 0] = 0;
    a.header[4 * tid + 1] = (int)(tot < a.max_items ? tot : a.max_items);
    a.header[4 * tid + 2] = 0;
    a.header[4 * tid + 3] = 0;
  }
  for (int g = tid; g < ntiles; g += kSchedThreads) {
    int b, t, L, U, wave;
    tile_of(g, b, t, L, U, wave);
    const int c0 = tile_count(key_tiles_of_query_tile(t, L, U));
    const int c1 = tile_count(query_tiles_of_key_tile(t, L, U));
    const int pos0 = atomicAdd(&hist[0][key_of(wave, c0)], a.H);
    const int pos1 = atomicAdd(&hist[1][key_of(wave, c1)], a.H);
    for (int h = 0; h < a.H; ++h) {
      if (pos0 + h < a.max_items) a.dq_items[pos0 + h] = make_int4(b, t, h, c0);
      if (pos1 + h < a.max_items) a.kv_items[pos1 + h] = make_int4(b, t, h, c1);
    }
  }
}

}  // namespace hstu
