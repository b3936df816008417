// schedule.cuh — tile geometry of the target-aware mask and the device-side work-list builder.
//
// Mask (DLRMv3 review, section "model selection": history encoded once and shared by every
// candidate; infolabhq.com multi-stage page: the user side never depends on a candidate, and
// target-aware attention weighs the history against each candidate):
//   query at position i of a segment with U history tokens may see key j iff
//     i <  U : j <= i                 (history token, causal over the history)
//     i >= U : j <  U  or  j == i     (candidate: all history, then itself)
// The keys visible to a block of queries at positions [p0, p1) are therefore
//     [0, p1)                         if p1 <= U
//     [0, U)  +  [max(p0, U), p1)     otherwise,
// i.e. at most two runs of 128-key tiles.  Tiles outside them are never enumerated.
#pragma once

#include <cstdint>

namespace hstu {

constexpr int kTileRows = 128;  // query rows per half / keys per key tile
constexpr int kItemRows = 128;  // query rows per work item: one query tile

__host__ __device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }

// Key tiles [0, e1) followed by [s2, e2), with s2 >= e1 (an empty second run has s2 == e2).
struct TileRange {
  int e1, s2, e2;
};

__host__ __device__ __forceinline__ TileRange key_tiles(int p0, int p1, int U) {
  TileRange r{0, 0, 0};
  if (p1 <= p0) return r;
  if (p1 <= U) {
    r.e1 = cdiv(p1, kTileRows);
    r.s2 = r.e2 = r.e1;
    return r;
  }
  r.e1 = cdiv(U, kTileRows);
  const int s = (p0 > U ? p0 : U) / kTileRows;
  const int e = cdiv(p1, kTileRows);
  if (s <= r.e1) {
    r.e1 = (e > r.e1) ? e : r.e1;
    r.s2 = r.e2 = r.e1;
  } else {
    r.s2 = s;
    r.e2 = e;
  }
  return r;
}

__host__ __device__ __forceinline__ int tile_count(const TileRange& r) { return r.e1 + (r.e2 - r.s2); }
__host__ __device__ __forceinline__ int tile_at(const TileRange& r, int idx) {
  return idx < r.e1 ? idx : r.s2 + (idx - r.e1);
}
__host__ __device__ __forceinline__ bool tile_in(const TileRange& r, int t) {
  return t < r.e1 || (t >= r.s2 && t < r.e2);
}

// Score tiles computed by one work item: query rows [128*blk, 128*blk + nrows) at positions
// pos0.. of a segment with U history tokens.
__host__ __device__ __forceinline__ int item_cost(int pos0, int nrows, int U) {
  return nrows > 0 ? tile_count(key_tiles(pos0, pos0 + nrows, U)) : 0;
}

constexpr unsigned kErrBadOffsets = 1u;
constexpr unsigned kErrTimeout = 2u;

constexpr int kSchedThreads = 256;
constexpr int kSchedWarps = kSchedThreads / 32;
constexpr int kMaxCostBins = 4096;
constexpr int kCachedUsers = 256;  // batches up to this many users keep per-user values in shared memory

struct SchedArgs {
  const int32_t* seq_offsets;  // [B+1]
  const int32_t* num_targets;  // [B] or null
  const int32_t* cached_len;   // [B] or null
  int32_t B, H, total_kv, total_q, max_seq_len, nbins, max_items;
  // Users are taken in waves by their first key row (wave = row / wave_rows, at most nwaves - 1),
  // each wave's K and V about a fixed share of L2; waves run in order, items by cost within one.
  int32_t wave_rows, nwaves;
  int32_t* q_start;       // [B] out: first query row of each user, -1 if the user is skipped
  int32_t* block_start;    // [B+1] out: index of each user's first 128-row block among all blocks
  int4* items;            // [max_items] out: {b, pair, h, cost}, non-increasing cost
  int32_t* num_items;     // [1] out
  int32_t* work_counter;  // [1] out: reset to 0 for the attention kernel's dynamic scheduler
  int32_t* done_counter;  // [1] out: reset to 0 (CTAs of the attention kernel that finished)
  unsigned* err;          // device error word
};

// Inclusive block-wide prefix sums of two values per thread (kSchedThreads threads); also
// returns the block totals.  `scratch` holds 2 x 32 values.
__device__ __forceinline__ void block_inclusive_scan2(long long& a, long long& b, long long (*scratch)[32],
                                                      long long& total_a, long long& total_b) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long na = __shfl_up_sync(0xffffffffu, a, o);
    const long long nb = __shfl_up_sync(0xffffffffu, b, o);
    if (lane >= o) {
      a += na;
      b += nb;
    }
  }
  if (lane == 31) {
    scratch[0][warp] = a;
    scratch[1][warp] = b;
  }
  __syncthreads();
  if (warp == 0) {
    long long wa = lane < kSchedWarps ? scratch[0][lane] : 0, wb = lane < kSchedWarps ? scratch[1][lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long na = __shfl_up_sync(0xffffffffu, wa, o);
      const long long nb = __shfl_up_sync(0xffffffffu, wb, o);
      if (lane >= o) {
        wa += na;
        wb += nb;
      }
    }
    scratch[0][lane] = wa;
    scratch[1][lane] = wb;
  }
  __syncthreads();
  if (warp > 0) {
    a += scratch[0][warp - 1];
    b += scratch[1][warp - 1];
  }
  total_a = scratch[0][kSchedWarps - 1];
  total_b = scratch[1][kSchedWarps - 1];
  __syncthreads();
}

// Inclusive block-wide prefix sum of one value per thread (kSchedThreads threads); also
// returns the block total.  `scratch` holds 32 values.
__device__ __forceinline__ long long block_inclusive_scan(long long v, long long* scratch,
                                                          long long* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    long long n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) scratch[warp] = v;
  __syncthreads();
  if (warp == 0) {
    long long w = lane < kSchedWarps ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      long long n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    scratch[lane] = w;
  }
  __syncthreads();
  if (warp > 0) v += scratch[warp - 1];
  *total = scratch[kSchedWarps - 1];
  __syncthreads();
  return v;
}

// User owning block g: the last b with block_start[b] <= g (users without blocks share a start).
// block_start may live in shared or global memory.
__device__ __forceinline__ int owner_of(const int32_t* block_start, int B, int g) {
  int lo = 0, hi = B;  // block_start[lo] <= g < block_start[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (block_start[mid] <= g) lo = mid; else hi = mid;
  }
  return lo;
}

// One CTA of kSchedThreads threads.  Validates every user, assigns query-row starts, and writes
// the work items wave by wave, each wave's items by non-increasing cost (counting sort over
// (wave, cost) keys; ties in any order).  A wave is the users whose first key row falls in one
// window of wave_rows rows: so the K and V tiles that the CTAs running at one time share stay in
// L2, instead of every user's tiles being fetched again for each cost level.  A batch whose K and
// V fit the window is one wave, ordered by cost alone.  The per-block passes run one thread per
// (user, 128-row block).
__global__ void __launch_bounds__(kSchedThreads) schedule_kernel(const SchedArgs a) {
  // A dependent attention kernel may start its prologue now; it waits for this grid's writes
  // (griddepcontrol.wait) before it reads anything in global memory.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ int hist[kMaxCostBins];
  __shared__ long long scan_scratch[2][32];
  __shared__ long long carry_q, carry_p;
  // Per-user values of pass 1, kept on chip for passes 2 and 4 when the batch is small enough
  // (their reads are then shared-memory latency instead of a chain of global loads).
  __shared__ int s_L[kCachedUsers], s_U[kCachedUsers], s_c[kCachedUsers], s_q[kCachedUsers], s_w[kCachedUsers];
  __shared__ int s_ps[kCachedUsers + 1];
  const bool cached = a.B <= kCachedUsers;
  const int tid = threadIdx.x;
  const int nbins = a.nbins;
  const int nkeys = nbins * a.nwaves;  // <= kMaxCostBins (host)

  for (int i = tid; i < nkeys; i += kSchedThreads) hist[i] = 0;
  if (tid == 0) {
    carry_q = 0;
    carry_p = 0;
  }
  __syncthreads();

  // Pass 1: per-user validation; one scan gives both the query-row starts (the caller's layout)
  // and the block starts.  Lengths are taken in 64 bits, so that corrupt offsets cannot wrap.
  for (int base = 0; base < a.B; base += kSchedThreads) {
    const int b = base + tid;
    long long nq = 0, nblocks = 0;  // rows in the layout; 128-row blocks to compute
    bool ok = false;
    int L = 0, T = 0, c = 0;
    if (b < a.B) {
      const int o0 = a.seq_offsets[b], o1 = a.seq_offsets[b + 1];
      const long long L64 = (long long)o1 - o0;
      T = a.num_targets ? a.num_targets[b] : 0;
      c = a.cached_len ? a.cached_len[b] : 0;
      ok = o0 >= 0 && L64 >= 0 && o1 <= a.total_kv && L64 <= a.max_seq_len && T >= 0 && T <= L64 && c >= 0 &&
           c <= L64 - T;
      if (b == 0 && o0 != 0) ok = false;
      if (b == a.B - 1 && o1 != a.total_kv) ok = false;
      if (!ok) atomicOr(a.err, kErrBadOffsets);
      L = ok ? (int)L64 : 0;
      // A skipped user still owns its rows of the layout, so later users keep their places; a
      // corrupt length is capped, and the layout check below then skips what follows it.
      const long long cc = c < 0 ? 0 : c;
      nq = L64 > cc ? L64 - cc : 0;
      if (nq > (long long)a.total_q + 1) nq = (long long)a.total_q + 1;
      nblocks = ok ? cdiv(L - c, kItemRows) : 0;
    }
    long long incl_q = nq, incl_p = nblocks, tot_q, tot_p;
    block_inclusive_scan2(incl_q, incl_p, scan_scratch, tot_q, tot_p);
    const long long start_q = carry_q + incl_q - nq;
    const long long start_p = carry_p + incl_p - nblocks;
    if (b < a.B) {
      if (ok && (start_q < 0 || start_q + nq > a.total_q)) {
        ok = false;
        atomicOr(a.err, kErrBadOffsets);
      }
      a.q_start[b] = ok ? (int)start_q : -1;
      a.block_start[b] = (int)start_p;
      if (cached) {
        s_L[b] = L;
        s_U[b] = L - T;
        s_c[b] = c;
        s_q[b] = ok ? (int)start_q : -1;
        s_ps[b] = (int)start_p;
        s_w[b] = ok ? min(a.seq_offsets[b] / a.wave_rows, a.nwaves - 1) : 0;
      }
    }
    __syncthreads();
    if (tid == 0) {
      carry_q += tot_q;
      carry_p += tot_p;
    }
    __syncthreads();
  }
  const int nblocks_total = (int)carry_p;
  if (tid == 0) {
    a.block_start[a.B] = nblocks_total;
    if (cached) s_ps[a.B] = nblocks_total;
    if (carry_q != a.total_q) atomicOr(a.err, kErrBadOffsets);
  }
  __syncthreads();
  // Cost of block g (and its user), from shared memory when cached; `key` orders the items: its
  // wave first, then non-increasing cost.
  auto block_of = [&](int g, int& b, int& pr, int& cost, int& key) {
    b = owner_of(cached ? s_ps : a.block_start, a.B, g);
    if ((cached ? s_q[b] : a.q_start[b]) < 0) return false;
    const int L = cached ? s_L[b] : a.seq_offsets[b + 1] - a.seq_offsets[b];
    const int U = cached ? s_U[b] : L - (a.num_targets ? a.num_targets[b] : 0);
    const int c = cached ? s_c[b] : (a.cached_len ? a.cached_len[b] : 0);
    pr = g - (cached ? s_ps[b] : a.block_start[b]);
    const int rows = (L - c) - pr * kItemRows;
    cost = item_cost(c + pr * kItemRows, rows < kItemRows ? rows : kItemRows, U);
    const int wave = cached ? s_w[b] : min(a.seq_offsets[b] / a.wave_rows, a.nwaves - 1);
    key = wave * nbins + (nbins - 1 - (cost < nbins ? cost : nbins - 1));
    return true;
  };

  // Pass 2: key histogram, one thread per block.
  for (int g = tid; g < nblocks_total; g += kSchedThreads) {
    int b, pr, cost, key;
    if (!block_of(g, b, pr, cost, key)) continue;
    atomicAdd(&hist[key], a.H);
  }
  __syncthreads();

  // Pass 3: key start = number of items with smaller keys.
  const int per = cdiv(nkeys, kSchedThreads);
  long long part = 0;
  for (int k = 0; k < per; ++k) {
    const int key = tid * per + k;
    if (key < nkeys) part += hist[key];
  }
  __syncthreads();
  long long tot;
  const long long incl = block_inclusive_scan(part, scan_scratch[0], &tot);
  long long run = incl - part;
  for (int k = 0; k < per; ++k) {
    const int key = tid * per + k;
    if (key < nkeys) {
      const int n = hist[key];
      hist[key] = (int)run;
      run += n;
    }
  }
  __syncthreads();
  if (tid == 0) {
    *a.num_items = (int)(tot < a.max_items ? tot : a.max_items);
    *a.work_counter = 0;
    *a.done_counter = 0;
  }

  // Pass 4: scatter the items into their keys' ranges, one thread per block.
  for (int g = tid; g < nblocks_total; g += kSchedThreads) {
    int b, pr, cost, key;
    if (!block_of(g, b, pr, cost, key)) continue;
    const int pos = atomicAdd(&hist[key], a.H);
    for (int h = 0; h < a.H; ++h)
      if (pos + h < a.max_items) a.items[pos + h] = make_int4(b, pr, h, cost);
  }
}

}  // namespace hstu
