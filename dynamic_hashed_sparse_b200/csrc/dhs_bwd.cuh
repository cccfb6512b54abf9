// Backward kernels: probe, group-by-row (LSD radix sort of (row, bag) pairs),
// fp64 segment reduce and the fused row optimizer.
//
// The gradient of sum pooling sends each bag's output gradient to every id of
// the bag; a row's gradient is the sum over its occurrences (RecIS overview,
// code layout: a fused sparse-gradient update kernel with fewer atomics; DLRM
// explainer, pitfall 4: a sparse optimizer touches only the rows of the
// batch).  Occurrences are grouped by a stable sort on the row offset, so
// each row's gradient is summed in batch order by one owner and written once:
// there are no per-element atomics on rows.  A row whose run spans three or
// more sort chunks (a hot key) is summed in pieces by every chunk it covers;
// the pieces are then added in batches and the batch sums in a fixed order.
#pragma once

#include <climits>

#include "dhs_device.cuh"

// Tuning constants (compile-time; -D overrides them when sweeping):
//   DHS_SEG_PREFETCH  1: the segment kernel prefetches into L2 the table row of
//                     each segment that opens among the pairs in flight; 0: not
//   DHS_RADIX_ITEMS   keys per thread in a radix-sort tile
#ifndef DHS_SEG_PREFETCH
#define DHS_SEG_PREFETCH 0
#endif
#ifndef DHS_RADIX_ITEMS
#define DHS_RADIX_ITEMS 16
#endif
//   DHS_SEG_MINB      resident 256-thread blocks per SM the segment kernel is
//                     compiled for (register budget) when a lane holds one
//                     float4 column
#ifndef DHS_SEG_MINB
#define DHS_SEG_MINB 3
#endif
//   DHS_SEG_RING      gradient rows in flight per group (shared-memory ring)
//                     for a row of <= 128 floats; wider rows use fewer
#ifndef DHS_SEG_RING
#define DHS_SEG_RING 8
#endif
//   DHS_RADIX_MINB    resident blocks per SM the one-sweep radix pass is
//                     compiled for (register budget)
//   DHS_SEGW_MIN_DIM  rows of at least this many floats use the warp-per-chunk
//                     segment kernel; narrower rows the lane-group kernel
#ifndef DHS_SEGW_MIN_DIM
#define DHS_SEGW_MIN_DIM 32
#endif
//   DHS_SEG_NARROW_MAX_DIM, DHS_SEG_NARROW_RUN  fp32 rows of more than
//                     DHS_SEGW_MIN_DIM and at most DHS_SEG_NARROW_MAX_DIM
//                     floats use the lane-group kernel while the table's
//                     backward calls have averaged fewer than
//                     DHS_SEG_NARROW_RUN ids per distinct row
#ifndef DHS_SEG_NARROW_MAX_DIM
#define DHS_SEG_NARROW_MAX_DIM 64
#endif
#ifndef DHS_SEG_NARROW_RUN
#define DHS_SEG_NARROW_RUN 8
#endif
//   DHS_SEGW_MINB     resident blocks per SM the warp segment kernel is
//                     compiled for (register budget) with up to 4 columns per
//                     lane; DHS_SEGW_BATCH4 gradient rows a warp stages per
//                     batch at 4 columns per lane (two batches in flight)
#ifndef DHS_SEGW_MINB
#define DHS_SEGW_MINB 3
#endif
#ifndef DHS_SEGW_BATCH4
#define DHS_SEGW_BATCH4 8
#endif
//   DHS_SEGW_REVERSE  1: the warp segment kernel takes its chunks from the
//                     last to the first; 0: in order
#ifndef DHS_SEGW_REVERSE
#define DHS_SEGW_REVERSE 1
#endif
//   DHS_SEGW_EVICT_FIRST 1: gradient rows of calls with about one id per bag
//                     are staged with an L2 evict-first policy; 0: normal
#ifndef DHS_SEGW_EVICT_FIRST
#define DHS_SEGW_EVICT_FIRST 1
#endif
#ifndef DHS_RADIX_MINB
#define DHS_RADIX_MINB 3
#endif
//   DHS_SEG_RUN_TABLE 1: long segments are finished by the segment kernel's
//                     warp that brings the last piece; 0: all go to the
//                     combine kernels
#ifndef DHS_SEG_RUN_TABLE
#define DHS_SEG_RUN_TABLE 1
#endif
//   DHS_SEG_RUN_TABLE_NARROW the same for the lane-group segment kernel
#ifndef DHS_SEG_RUN_TABLE_NARROW
#define DHS_SEG_RUN_TABLE_NARROW 1
#endif
//   DHS_SEG_FINISH_PIECES pieces of a long segment the segment kernel's warp
//                     adds itself (longer ones go to the combine kernels)
#ifndef DHS_SEG_FINISH_PIECES
#define DHS_SEG_FINISH_PIECES 32
#endif
//   DHS_PROBE_DEDUP   1: the backward probe probes a key held by several lanes
//                     of a warp once (match.any); 0: every lane probes
#ifndef DHS_PROBE_DEDUP
#define DHS_PROBE_DEDUP 0
#endif
//   DHS_RADIX_MATCH   how a radix pass finds the lanes of equal digit:
//                     0 match.any when the warp's first 32 items hold at most
//                     DHS_RADIX_MATCH_DISTINCT distinct digits, else one
//                     ballot per digit bit; 1 match.any always; 2 ballots
//                     always
#ifndef DHS_RADIX_MATCH
#define DHS_RADIX_MATCH 0
#endif
#ifndef DHS_RADIX_MATCH_DISTINCT
#define DHS_RADIX_MATCH_DISTINCT 16
#endif
//   DHS_LOOKBACK_WINDOW predecessor tiles a radix pass's look-back reads at once
//   DHS_BWD_RECORD   1: the backward probe reads the rows a split forward
//                    recorded per position where the keys are the same; 0:
//                    it always probes the IDMap
#ifndef DHS_BWD_RECORD
#define DHS_BWD_RECORD 1
#endif
#ifndef DHS_LOOKBACK_WINDOW
#define DHS_LOOKBACK_WINDOW 8
#endif

namespace dhs {

// ---------------------------------------------------------------------------
// probe: (row, bag) of every position, bag-major order
// ---------------------------------------------------------------------------

#ifndef DHS_TEMPLATES_ONLY
// ---------------------------------------------------------------------------
// LSD radix sort of 32-bit keys with 32-bit values, 8-bit digits, stable,
// one kernel per digit pass (decoupled look-back across tiles)
// ---------------------------------------------------------------------------
constexpr int kRadixThreads = 256;
constexpr int kRadixItems = DHS_RADIX_ITEMS;
constexpr int kRadixWarpItems = 32 * kRadixItems;
constexpr int kRadixTile = kRadixWarpItems * (kRadixThreads / 32);
constexpr int kRadixBins = 256;
constexpr int kRadixMaxPasses = 4;
constexpr unsigned long long kLbAggregate = 1ull << 62;  // tile count published
constexpr unsigned long long kLbPrefix = 2ull << 62;     // inclusive prefix published
constexpr unsigned long long kLbCountMask = (1ull << 62) - 1;
constexpr unsigned kLookbackSpins = 1u << 22;  // bounded wait for a predecessor tile
constexpr int kLookbackWindow = DHS_LOOKBACK_WINDOW;  // predecessors read per look-back step
constexpr int kRadixMatchDistinct = DHS_RADIX_MATCH_DISTINCT;
// the counters a backward starts from zero (cleared by the previous
// backward's probe, or by a memset before the allocation-free backward's):
// digit histograms of every pass, one tile counter per pass, the segment
// kernel's chunk counter, the count of long-segment owner chunks and the
// combine's batch and slot counters
constexpr int kSortZeroWords = kRadixMaxPasses * kRadixBins + kRadixMaxPasses + 4;
constexpr int kSegChunkCtrWord = kRadixMaxPasses * kRadixBins + kRadixMaxPasses;
constexpr int kSegOwnerCtrWord = kSegChunkCtrWord + 1;
constexpr int kCombineBatchCtrWord = kSegChunkCtrWord + 2;
constexpr int kCombineSlotCtrWord = kSegChunkCtrWord + 3;

// Warp per chunk of bpc bags (64 when bags are short, 32 when they are long,
// so that long bags still spread over enough warps); positions 64 at a time,
// two per lane, so that each lane has two probes in flight.  A position's bag
// is the number of the chunk's bag ends at or before it (a binary search over
// the ends held in the lanes' registers).  Missing or negative keys get row
// `sentinel` (sorted last, never updated).
// rec_keys / rec_rows (both null, or both set): the last forward's keys and
// rows per position (a split forward over the same number of positions);
// a position whose key equals the recorded one takes the recorded row
// without probing the IDMap.
// Extended pooling (per-sample weights psw, or mean pooling): the sort value
// is the position instead of the bag; bagpos[p] = its bag and mult[p] = its
// weight psw[p] (the bag's gradient is multiplied by it) or, for mean
// pooling, the bag's length (the gradient is divided by it).
template <bool EXT>
__global__ void __launch_bounds__(256, 4)
bwd_probe_kernel(IdMap m, const long long* __restrict__ keys, long long n_keys,
                 const long long* __restrict__ bag_off, long long n_bags,
                 unsigned* __restrict__ rkey, unsigned* __restrict__ rval, unsigned sentinel,
                 unsigned* __restrict__ hist, int passes, unsigned long long* __restrict__ status0,
                 long long status0_words, unsigned* __restrict__ zero32, long long zero32_words,
                 unsigned* __restrict__ next_ctr, long long next_ctr_words, int bpc,
                 const float* __restrict__ psw, bool mean, unsigned* __restrict__ bagpos,
                 double* __restrict__ mult, const long long* __restrict__ rec_keys,
                 const long long* __restrict__ rec_rows, DevState* st) {
  pdl_enter();
  constexpr bool ext = EXT;
  constexpr unsigned FULL = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  // the sort's digit counts of every pass, taken here from the rows this
  // kernel writes (hist is zero on entry); the first pass's look-back words
  // and the segment kernel's arrival table (zero32) cleared, and the counters
  // of the next backward (next_ctr, another area than this one's)
  __shared__ unsigned h[kRadixMaxPasses][kRadixBins];
  for (int i = threadIdx.x; i < kRadixMaxPasses * kRadixBins; i += blockDim.x) (&h[0][0])[i] = 0u;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < status0_words;
       i += (long long)gridDim.x * blockDim.x)
    status0[i] = 0ull;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < zero32_words;
       i += (long long)gridDim.x * blockDim.x)
    zero32[i] = 0u;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < next_ctr_words;
       i += (long long)gridDim.x * blockDim.x)
    next_ctr[i] = 0u;
  __syncthreads();
  auto count = [&](unsigned k) {
    for (int ps = 0; ps < passes; ++ps) atomicAdd(&h[ps][(k >> (8 * ps)) & 255u], 1u);
  };
  // positions and bags fit in 31 bits (the host rejects larger calls)
  const int n = (int)n_keys;
  const long long nchunks = (n_bags + bpc - 1) / bpc;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long c = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; c < nchunks;
       c += nw) {
    // a chunk of bpc (32 or 64) bags: lane l holds the ends of bags b0 + l and
    // b0 + 32 + l
    const long long b0 = c * bpc;
    const int nb = (int)min((long long)bpc, n_bags - b0);
    long long s64 = __ldg(bag_off + b0);
    long long x0 = lane < nb ? __ldg(bag_off + b0 + lane + 1) : n_keys;
    long long x1 = lane + 32 < nb ? __ldg(bag_off + b0 + lane + 33) : n_keys;
    bool bad = (b0 == 0 && s64 != 0) || s64 < 0 || s64 > n_keys;
    s64 = s64 < 0 ? 0 : (s64 > n_keys ? n_keys : s64);
    if (lane < nb && (x0 < s64 || x0 > n_keys || (b0 + lane + 1 == n_bags && x0 != n_keys))) bad = true;
    if (lane + 32 < nb && (x1 < s64 || x1 > n_keys || (b0 + lane + 33 == n_bags && x1 != n_keys))) bad = true;
    int s = (int)s64;
    int e0 = (int)(x0 < s64 ? s64 : (x0 > n_keys ? n_keys : x0));
    int e1 = (int)(x1 < s64 ? s64 : (x1 > n_keys ? n_keys : x1));
    // running max, so that ends never decrease along the chunk
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(FULL, e0, o);
      if (lane >= o && y > e0) {
        e0 = y;
        bad = true;
      }
    }
    {
      const int carry = __shfl_sync(FULL, e0, 31);
      if (carry > e1) {
        e1 = carry;
        if (lane + 32 < nb) bad = true;
      }
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(FULL, e1, o);
      if (lane >= o && y > e1) {
        e1 = y;
        bad = true;
      }
    }
    // every position must get a (row, bag) pair even when the offsets are
    // malformed: the first bag starts at 0 and the last one ends at n_keys
    if (b0 == 0) s = 0;
    if (b0 + nb == n_bags) {
      if (lane == nb - 1) e0 = n;
      if (lane + 32 == nb - 1) e1 = n;
    }
    // one id per bag throughout the chunk (a common case): a position's bag
    // is its offset from the chunk's start, no search needed
    const bool singles =
        __all_sync(FULL, (lane >= nb || e0 == s + lane + 1) && (lane + 32 >= nb || e1 == s + lane + 33));
    if (lane >= nb) e0 = INT_MAX;
    if (lane + 32 >= nb) e1 = INT_MAX;
    if (bad) latch(st, kErrInvalid);
    const int E = nb > 32 ? __shfl_sync(FULL, e1, nb - 33) : __shfl_sync(FULL, e0, nb - 1);
    // bag of position p: the number of bag ends <= p (binary search over the 64)
    auto bag_of = [&](int p) -> int {
      int lo = 0;
#pragma unroll
      for (int step = 32; step >= 1; step >>= 1) {
        const int j = lo + step - 1;
        const int a0 = __shfl_sync(FULL, e0, j & 31);
        const int a1 = __shfl_sync(FULL, e1, j & 31);
        if ((j < 32 ? a0 : a1) <= p) lo += step;
      }
      return lo;
    };
    for (int ws = s; ws < E; ws += 64) {
      const int p0 = ws + lane, p1 = ws + 32 + lane;
      // both positions' keys and probes are in flight together
      const long long k0 = p0 < E ? __ldg(keys + p0) : 0;
      const long long k1 = p1 < E ? __ldg(keys + p1) : 0;
      long long f0 = -1, f1 = -1;
      if (rec_keys) {
        // the forward's record of these positions: where its key is this
        // key, its row (or no row) stands, and only other keys are probed
        const long long q0 = p0 < E ? __ldg(rec_keys + p0) : 0, r0 = p0 < E ? __ldg(rec_rows + p0) : 0;
        const long long q1 = p1 < E ? __ldg(rec_keys + p1) : 0, r1 = p1 < E ? __ldg(rec_rows + p1) : 0;
        if (p0 < E && k0 >= 0)
          f0 = q0 == k0 && r0 >= 0 ? r0 : (q0 == k0 && r0 == kRecNoRow ? -2 : probe_find(m, (unsigned long long)k0));
        if (p1 < E && k1 >= 0)
          f1 = q1 == k1 && r1 >= 0 ? r1 : (q1 == k1 && r1 == kRecNoRow ? -2 : probe_find(m, (unsigned long long)k1));
      } else {
#if DHS_PROBE_DEDUP
      // a key held by several lanes is probed once, by the lowest of them
      const unsigned long long q0 = p0 < E && k0 >= 0 ? (unsigned long long)k0 : ~0ull;
      const unsigned long long q1 = p1 < E && k1 >= 0 ? (unsigned long long)k1 : ~0ull;
      const unsigned m0 = __match_any_sync(FULL, q0), m1 = __match_any_sync(FULL, q1);
      const int l0 = __ffs(m0) - 1, l1 = __ffs(m1) - 1;
      if (l0 == lane && q0 != ~0ull) f0 = probe_find(m, q0);
      if (l1 == lane && q1 != ~0ull) f1 = probe_find(m, q1);
      f0 = __shfl_sync(FULL, f0, l0);
      f1 = __shfl_sync(FULL, f1, l1);
#else
      if (p0 < E && k0 >= 0) f0 = probe_find(m, (unsigned long long)k0);
      if (p1 < E && k1 >= 0) f1 = probe_find(m, (unsigned long long)k1);
#endif
      }
      const int g0 = singles ? p0 - s : bag_of(p0), g1 = singles ? p1 - s : bag_of(p1);
      // f < 0: no row (-1 absent: an error; -2 known but not admitted: skipped)
      if (p0 < E) {
        if (k0 < 0) latch(st, kErrInvalid);
        else if (f0 == -1) latch(st, kErrNotFound);
        rkey[p0] = f0 >= 0 ? (unsigned)f0 : sentinel;
        rval[p0] = ext ? (unsigned)p0 : (unsigned)(b0 + g0);
        count(f0 >= 0 ? (unsigned)f0 : sentinel);
      }
      if (p1 < E) {
        if (k1 < 0) latch(st, kErrInvalid);
        else if (f1 == -1) latch(st, kErrNotFound);
        rkey[p1] = f1 >= 0 ? (unsigned)f1 : sentinel;
        rval[p1] = ext ? (unsigned)p1 : (unsigned)(b0 + g1);
        count(f1 >= 0 ? (unsigned)f1 : sentinel);
      }
      if constexpr (EXT) {
        // bag g of the chunk spans [end(g - 1), end(g)), end(-1) = s
        auto bag_end = [&](int g) -> int {
          const int a0 = __shfl_sync(FULL, e0, g & 31);
          const int a1 = __shfl_sync(FULL, e1, g & 31);
          return g < 32 ? a0 : a1;
        };
        // every lane takes part in every shuffle (no shuffle under a condition)
        const int end0 = bag_end(g0), prev0 = bag_end(max(g0 - 1, 0));
        const int end1 = bag_end(g1), prev1 = bag_end(max(g1 - 1, 0));
        const int beg0 = g0 > 0 ? prev0 : s, beg1 = g1 > 0 ? prev1 : s;
        if (p0 < E) {
          bagpos[p0] = (unsigned)(b0 + g0);
          mult[p0] = psw ? (double)__ldg(psw + p0) : (double)(end0 - beg0);
        }
        if (p1 < E) {
          bagpos[p1] = (unsigned)(b0 + g1);
          mult[p1] = psw ? (double)__ldg(psw + p1) : (double)(end1 - beg1);
        }
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < passes * kRadixBins; i += blockDim.x) {
    const unsigned v = (&h[0][0])[i];
    if (v) atomicAdd(hist + i, v);
  }
}


// Block-wide exclusive scan of one value per thread (256 threads).
__device__ __forceinline__ unsigned block_exclusive_scan_256(unsigned x, unsigned* wsum,
                                                             unsigned& total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  unsigned inc = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) wsum[wid] = inc;
  __syncthreads();
  unsigned pre = 0;
  total = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const unsigned v = wsum[k];
    if (k < wid) pre += v;
    total += v;
  }
  __syncthreads();
  return pre + inc - x;
}

// One stable digit pass.  Tiles are numbered in the order blocks start (an
// atomic counter), so a tile only ever waits for tiles whose blocks are
// already running.  Each warp ranks its 32 x kRadixItems items in order
// (kRadixItems rounds of 32 lanes; the lanes of equal digit give the rank
// within a round, a per-warp shared counter carries it across rounds); the
// tile publishes its digit counts, adds up its predecessors' (decoupled
// look-back), publishes its inclusive prefix, places its items in digit order
// in shared memory and writes them out in runs.  A wait that exceeds its
// bound latches kErrInternal and the pass goes on (its output is then
// undefined, never out of bounds).
__global__ void __launch_bounds__(kRadixThreads, DHS_RADIX_MINB)
radix_onesweep_kernel(const unsigned* __restrict__ kin, const unsigned* __restrict__ vin,
                      unsigned* __restrict__ kout, unsigned* __restrict__ vout, long long n,
                      int shift, const unsigned* __restrict__ hist,
                      unsigned long long* __restrict__ status, unsigned* __restrict__ tile_ctr,
                      unsigned long long* __restrict__ next_status, long long next_words, DevState* st) {
  pdl_enter();
  __shared__ unsigned s_k[kRadixTile];
  __shared__ unsigned s_v[kRadixTile];
  __shared__ unsigned wc[8][kRadixBins + 1];
  __shared__ unsigned dstart[kRadixBins];
  __shared__ unsigned gbase[kRadixBins];
  __shared__ unsigned wsum[8];
  __shared__ unsigned s_tile;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (threadIdx.x == 0) s_tile = atomicAdd(tile_ctr, 1u);
  // the next pass's look-back words start at zero (that pass runs after this one)
  for (long long i = (long long)blockIdx.x * kRadixThreads + threadIdx.x; i < next_words;
       i += (long long)gridDim.x * kRadixThreads)
    next_status[i] = 0ull;
  for (int i = threadIdx.x; i < 8 * (kRadixBins + 1); i += kRadixThreads) (&wc[0][0])[i] = 0;
  __syncthreads();
  // positions fit in 31 bits (the host rejects larger calls)
  const int tile = (int)s_tile;
  const int tile0 = tile * kRadixTile;
  const int tile_n = max(0, min(kRadixTile, (int)n - tile0));
  // items r * 32 + lane of this warp are in range below rem
  const int rem = tile_n - wid * kRadixWarpItems;

  // keys now; values only when they are placed (fewer registers held)
  unsigned k[kRadixItems], lr[kRadixItems];
  const unsigned* kb = kin + tile0 + wid * kRadixWarpItems + lane;
  const unsigned* vb = vin + tile0 + wid * kRadixWarpItems + lane;
#pragma unroll
  for (int r = 0; r < kRadixItems; ++r) k[r] = r * 32 + lane < rem ? __ldg(kb + r * 32) : 0u;
  const unsigned lt = lanemask_lt();
  // the lanes of equal digit: match.any costs about as many steps as there
  // are distinct digits among the 32 lanes, one ballot per digit bit a fixed
  // nine; the number of distinct digits in the warp's first round decides
  // for all its rounds
  bool use_match = DHS_RADIX_MATCH == 1;
  if (DHS_RADIX_MATCH == 0) {
    const unsigned d0 = lane < rem ? ((k[0] >> shift) & 255u) : 256u;
    const unsigned p0 = __match_any_sync(0xffffffffu, d0);
    const int distinct = __popc(__ballot_sync(0xffffffffu, (__ffs(p0) - 1) == lane));
    use_match = distinct <= kRadixMatchDistinct;
  }
#pragma unroll
  for (int r = 0; r < kRadixItems; ++r) {
    const unsigned d = r * 32 + lane < rem ? ((k[r] >> shift) & 255u) : 256u;
    // (9 bits: 256 marks an item past the end)
    unsigned peers;
    if (use_match) {
      peers = __match_any_sync(0xffffffffu, d);
    } else {
      peers = 0xffffffffu;
#pragma unroll
      for (int b = 0; b < 9; ++b) {
        const bool bit = (d >> b) & 1u;
        const unsigned m = __ballot_sync(0xffffffffu, bit);
        peers &= bit ? m : ~m;
      }
    }
    const unsigned before = wc[wid][d];
    lr[r] = before + __popc(peers & lt);
    __syncwarp();
    if ((__ffs(peers) - 1) == lane) wc[wid][d] = before + __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  const int d = threadIdx.x;
  unsigned cnt = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const unsigned t = wc[w][d];
    wc[w][d] = cnt;
    cnt += t;
  }
  // publish this tile's count of digit d at once; the tile's items go to
  // shared memory in digit order before the look-back, so that no item is
  // held in registers while it waits
  volatile unsigned long long* sp = status + (long long)tile * kRadixBins + d;
  if (tile == 0) {
    *sp = kLbPrefix | cnt;
  } else {
    *sp = kLbAggregate | cnt;
  }
  unsigned dpre;
  {
    unsigned tot;
    dpre = block_exclusive_scan_256(hist[d], wsum, tot);
    dstart[d] = block_exclusive_scan_256(cnt, wsum, tot);
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kRadixItems; ++r) {
    if (r * 32 + lane < rem) {
      const unsigned dd = (k[r] >> shift) & 255u;
      const unsigned pos = dstart[dd] + wc[wid][dd] + lr[r];
      s_k[pos] = k[r];
      s_v[pos] = __ldg(vb + r * 32);
    }
  }
  unsigned long long excl = 0;
  if (tile > 0) {
    // kLookbackWindow predecessors are read at once (independent loads in
    // flight together) and taken in order until a prefix, or a tile that has
    // not published yet, is met; tile 0 always publishes a prefix, so the
    // walk never passes it
    int t = tile - 1;
    unsigned spins = 0;
    for (;;) {
      unsigned long long sv[kLookbackWindow];
#pragma unroll
      for (int i = 0; i < kLookbackWindow; ++i)
        sv[i] = t - i >= 0 ? *(volatile unsigned long long*)(status + (long long)(t - i) * kRadixBins + d) : 0ull;
      int used = 0;
      bool done = false;
#pragma unroll
      for (int i = 0; i < kLookbackWindow; ++i) {
        if (!done && used == i && (sv[i] & (kLbPrefix | kLbAggregate))) {
          excl += sv[i] & kLbCountMask;
          if (sv[i] & kLbPrefix) done = true;
          else used = i + 1;
        }
      }
      if (done) break;
      t -= used;
      if (used == 0) {
        if (++spins > kLookbackSpins || t < 0) {
          latch(st, kErrInternal);
          break;
        }
        __nanosleep(32);
      }
    }
    *sp = kLbPrefix | (excl + cnt);
  }
  gbase[d] = dpre + (unsigned)excl;
  __syncthreads();
  for (int i = threadIdx.x; i < tile_n; i += kRadixThreads) {
    const unsigned key = s_k[i];
    const unsigned dd = (key >> shift) & 255u;
    const unsigned o = gbase[dd] + (unsigned)i - dstart[dd];
    // o < n for counts that match the items; malformed bag offsets (already
    // reported) can count a position twice, so the bound is checked
    if (o < (unsigned)n) {
      kout[o] = key;
      vout[o] = s_v[i];
    } else {
      latch(st, kErrInvalid);
    }
  }
}

#endif  // DHS_TEMPLATES_ONLY

// One occurrence's gradient term added in fp64 for extended pooling: x times
// the weight, or x divided by the bag length (mean), each operation rounded
// on its own (no fused multiply-add), as the plain definition computes it.
__device__ __forceinline__ double ext_add(double acc, float x, double f, bool mean) {
  return __dadd_rn(acc, mean ? __ddiv_rn((double)x, f) : __dmul_rn((double)x, f));
}

// ---------------------------------------------------------------------------
// optimizer step on one row (fp32, each operation rounded)
// ---------------------------------------------------------------------------
struct OptArgs {
  int opt;  // 0 SGD, 1 Adagrad, 2 Adam, 3 row-wise Adagrad
  float lr, eps, b1, b2, c1, c2, bc1, bc2;
};

__device__ __forceinline__ float sgd_w(float w, float g, float lr) {
  return __fsub_rn(w, __fmul_rn(lr, g));
}
// Adagrad: G += g*g ; w -= (lr*g) / (sqrt(G) + eps)
__device__ __forceinline__ void adagrad_step(float& w, float& G, float g, float lr, float eps) {
  G = __fadd_rn(G, __fmul_rn(g, g));
  w = __fsub_rn(w, __fdiv_rn(__fmul_rn(lr, g), __fadd_rn(__fsqrt_rn(G), eps)));
}
// Adam: m = b1 m + (1-b1) g ; v = b2 v + (1-b2) g^2 ;
//       w -= (lr * m/bc1) / (sqrt(v/bc2) + eps)
__device__ __forceinline__ void adam_step(float& w, float& m, float& v, float g,
                                          const OptArgs& o) {
  m = __fadd_rn(__fmul_rn(o.b1, m), __fmul_rn(o.c1, g));
  v = __fadd_rn(__fmul_rn(o.b2, v), __fmul_rn(o.c2, __fmul_rn(g, g)));
  const float mhat = __fdiv_rn(m, o.bc1);
  const float vhat = __fdiv_rn(v, o.bc2);
  w = __fsub_rn(w, __fdiv_rn(__fmul_rn(o.lr, mhat), __fadd_rn(__fsqrt_rn(vhat), o.eps)));
}

// Weight j of a row: fp32, or bf16 widened (wfl < dim).
__device__ __forceinline__ float load_w(const float* row, int j, bool bf16) {
  if (!bf16) return row[j];
  return __uint_as_float((unsigned)reinterpret_cast<const unsigned short*>(row)[j] << 16);
}
__device__ __forceinline__ void store_w(float* row, int j, float w, bool bf16) {
  if (!bf16)
    row[j] = w;
  else
    reinterpret_cast<__nv_bfloat16*>(row)[j] = __float2bfloat16_rn(w);
}

// Scalar form for one column j (used by the combine kernel); the state
// starts wfl floats into the row.
__device__ __forceinline__ void update_col(float* row, int dim, int wfl, int j, float g, const OptArgs& o,
                                           float rowwise_den) {
  const bool bf16 = wfl != dim;
  float w = load_w(row, j, bf16);
  if (o.opt == 0) {
    w = sgd_w(w, g, o.lr);
  } else if (o.opt == 1) {
    float G = row[wfl + j];
    adagrad_step(w, G, g, o.lr, o.eps);
    row[wfl + j] = G;
  } else if (o.opt == 2) {
    float m = row[wfl + j], v = row[wfl + dim + j];
    adam_step(w, m, v, g, o);
    row[wfl + j] = m;
    row[wfl + dim + j] = v;
  } else {
    w = __fsub_rn(w, __fdiv_rn(__fmul_rn(o.lr, g), rowwise_den));
  }
  store_w(row, j, w, bf16);
}

// ---------------------------------------------------------------------------
// segment reduce + update
// ---------------------------------------------------------------------------

// The part of one row a lane owns: float4 columns gl + q*G (q < NV) of the
// weights and of each per-element state array (Adagrad: G; Adam: m, v), plus
// the row accumulator of row-wise Adagrad.  Loaded when a segment opens, so
// the loads overlap the gradient sum; written back once when it closes.
__host__ __device__ constexpr int seg_state_arrays(int opt) { return opt == 1 ? 1 : (opt == 2 ? 2 : 0); }

template <int OPT, int NV>
struct RowBuf {
  static constexpr int NS = seg_state_arrays(OPT);
  float4 w[NV];
  float4 st[NS > 0 ? NS : 1][NV];
  float acc_row;

  __device__ __forceinline__ void load(const float* row, int dim, int gl, int G) {
    const int d4 = dim >> 2;
    const float4* r4 = reinterpret_cast<const float4*>(row);
#pragma unroll
    for (int q = 0; q < NV; ++q) {
      const int c4 = gl + q * G;
      if (c4 < d4) {
        w[q] = r4[c4];
#pragma unroll
        for (int k = 0; k < NS; ++k) st[k][q] = r4[(k + 1) * d4 + c4];
      }
    }
    if (OPT == 3) acc_row = row[dim];
  }

  // one optimizer step with the row gradient held in fp64 by this lane;
  // rowwise_sq = sum over the whole row of g^2 (row-wise Adagrad only)
  __device__ __forceinline__ void step_store(float* row, int dim, int gl, int G,
                                             const double (&acc)[NV][4], const OptArgs& o,
                                             double rowwise_sq) {
    const int d4 = dim >> 2;
    float4* r4 = reinterpret_cast<float4*>(row);
    float den = 0.f, Gn = 0.f;
    if (OPT == 3) {
      Gn = __fadd_rn(acc_row, (float)(rowwise_sq / (double)dim));
      den = __fadd_rn(__fsqrt_rn(Gn), o.eps);
    }
#pragma unroll
    for (int q = 0; q < NV; ++q) {
      const int c4 = gl + q * G;
      if (c4 >= d4) continue;
      float* wp = &w[q].x;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float g = (float)acc[q][e];
        if (OPT == 0) {
          wp[e] = sgd_w(wp[e], g, o.lr);
        } else if (OPT == 1) {
          adagrad_step(wp[e], (&st[0][q].x)[e], g, o.lr, o.eps);
        } else if (OPT == 2) {
          adam_step(wp[e], (&st[0][q].x)[e], (&st[NS - 1][q].x)[e], g, o);
        } else {
          wp[e] = __fsub_rn(wp[e], __fdiv_rn(__fmul_rn(o.lr, g), den));
        }
      }
      r4[c4] = w[q];
#pragma unroll
      for (int k = 0; k < NS; ++k) r4[(k + 1) * d4 + c4] = st[k][q];
    }
    if (OPT == 3 && gl == 0) row[dim] = Gn;
  }
};

// Arrival sums of long segments: see the segment kernel's close step.
constexpr unsigned kRunBias = 1u << 30;

// Entry of row in the arrival table (inserted when absent); ~0u after
// latching kErrInternal when the table is full (it is sized for every long
// segment of sorted input, so only a failed sort gets there).
__device__ __forceinline__ unsigned run_slot(const RunTable& rt, unsigned row, DevState* st) {
  unsigned h = (row * 0x9E3779B1u) & rt.mask;  // Fibonacci hashing of the row
  for (unsigned i = 0; i <= rt.mask; ++i) {
    const unsigned old = atomicCAS(rt.key + h, 0u, row + 1u);
    if (old == 0u || old == row + 1u) return h;
    h = (h + 1u) & rt.mask;
  }
  latch(st, kErrInternal);
  return ~0u;
}

// Gradient rows in flight per group (ring of shared-memory slots, filled by
// cp.async): DHS_SEG_RING for a row of <= 128 floats, fewer for wider rows,
// so that a 256-thread block uses the same shared memory at every width.
__host__ __device__ constexpr int seg_ring(int nv) { return DHS_SEG_RING / nv > 0 ? DHS_SEG_RING / nv : 1; }
__host__ __device__ constexpr size_t seg_smem_bytes(int G, int NV) {
  return (size_t)(256 / G) * seg_ring(NV) * NV * G * 16;
}

__device__ __forceinline__ void cp_async16(unsigned dst, const void* src, unsigned src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// A group of G lanes owns sort chunk c = [cC, cC + C).  It sums, in fp64 and
// in sorted (= batch) order, the gradients of every segment that starts in the
// chunk and applies the optimizer to that row once.  A segment that started
// in an earlier chunk is skipped unless it is "long" (spans >= 3 chunks), in
// which case this chunk's piece is written as a partial.  A segment that
// starts here and ends in the next chunk is finished here (short overrun); one
// that reaches chunk c + 2 is long: its piece up to the chunk end is written
// as the starting partial and bwd_combine_kernel finishes it.
// Piece modes: 0 skip (owned by the previous chunk), 1 long head piece,
// 2 owned short segment, 3 long segment starting here.
// Data movement: the gradient row of pair i + R is copied into the group's
// shared-memory ring (cp.async, each lane its own 16-byte columns, so no lane
// reads another's data and no barrier is needed) while pair i is added; when
// a segment starts among the pairs in flight, its table row is prefetched
// into L2, so the row load at the segment's open mostly hits L2.
// EXT: as in bwd_segw_kernel (positions as sort values, bags and factors
// gathered from bagpos and mult).
template <int G, int NV, int OPT, bool EXT>
__global__ void __launch_bounds__(256, NV <= 2 ? DHS_SEG_MINB : 1)
bwd_seg_kernel(const unsigned* __restrict__ skey, const unsigned* __restrict__ sval, long long n,
               const float* __restrict__ grad, long long n_bags, int dim, RowSpace rs, OptArgs oa,
               double* __restrict__ part_head, double* __restrict__ part_tail,
               int C, unsigned* __restrict__ chunk_ctr,
               unsigned* __restrict__ owners, unsigned* __restrict__ owner_ctr, DevState* st,
               const unsigned* __restrict__ bagpos, const double* __restrict__ mult, bool mean,
               RunTable rt) {
  pdl_enter();
  constexpr int R = seg_ring(NV);
  extern __shared__ float4 seg_ring_smem[];
  const int lane = threadIdx.x & 31;
  const int gl = lane & (G - 1);
  const int gw = lane / G;
  const unsigned gmask = (G == 32) ? 0xffffffffu : (((1u << G) - 1u) << (gw * G));
  const int grp = threadIdx.x / G;
  float4* ring = seg_ring_smem + (size_t)grp * R * NV * G;
  const unsigned ring_s = (unsigned)__cvta_generic_to_shared(ring);
  // positions and bags fit in 31 bits (the host rejects larger calls)
  const int n32 = (int)n;
  const unsigned nb32 = (unsigned)n_bags;
  const int nchunks = (n32 + C - 1) / C;
  const unsigned nrows = (unsigned)min(st->row_count, 0xffffffffull);
  const int d4 = dim >> 2;
  const int pstride = NV * G * 4;  // doubles per partial vector
  const unsigned row_bytes = (unsigned)rs.stride * 4u;
  unsigned nseg_total = 0;

  // chunks are handed out one at a time (a counter), so groups that meet
  // cheap chunks take more of them and none idles while others still work
  auto next_chunk = [&]() {
    int v = 0;
    if (gl == 0) v = (int)atomicAdd(chunk_ctr, 1u);
    return __shfl_sync(gmask, v, 0, G);
  };
  for (int c = next_chunk(); c < nchunks; c = next_chunk()) {
    const int start = c * C;
    const int end = min(n32, start + C);
    const int limit = min(n32, end + C);  // an owned segment ends before chunk c + 2
    unsigned nseg = 0;

    // the keys that decide who owns the chunk's first and last pieces
    const unsigned cur0 = __ldg(skey + start);
    const unsigned prev = start > 0 ? __ldg(skey + start - 1) : ~0u;
    const unsigned back2 = c >= 2 ? __ldg(skey + (c - 1) * C - 1) : ~0u;
    const unsigned fwd1 = (c + 1) * C < n32 ? __ldg(skey + (c + 1) * C) : ~0u;
    const int p2 = (c + 2) * C;
    const bool has2 = p2 < n32;
    const unsigned fwd2 = has2 ? __ldg(skey + p2) : ~0u;

    // ---- producer: gradient rows of pairs start, start + 1, ... into the ring
    int pf = start;          // next pair to copy
    int pws = start - G;     // start of the producer's window of pairs
    unsigned pk = 0u, pv = 0u, pprev = prev;
    auto produce = [&]() {
      if (pf < limit) {
        if (pf >= pws + G) {
          pws = pf;
          pk = pws + gl < n32 ? __ldg(skey + pws + gl) : 0u;
          pv = pws + gl < n32 ? __ldg(sval + pws + gl) : 0u;
          if (EXT && pws + gl < n32) pv = __ldg(bagpos + pv);  // position -> bag
        }
        const int t = pf - pws;
        const unsigned b = __shfl_sync(gmask, pv, t, G);
        const unsigned k = __shfl_sync(gmask, pk, t, G);
        const bool ok = b < nb32 && k < nrows;
        const float* src = grad + (size_t)(ok ? b : 0u) * dim;
        const unsigned slot = ring_s + (unsigned)(((pf - start) % R) * NV * G) * 16u;
#pragma unroll
        for (int q = 0; q < NV; ++q) {
          const int c4 = gl + q * G;
          cp_async16(slot + (unsigned)(q * G + gl) * 16u, src + (c4 < d4 ? c4 * 4 : 0),
                     ok && c4 < d4 ? 16u : 0u);
        }
        if (DHS_SEG_PREFETCH >= 1 && gl == 0 && ok && k != pprev) prefetch_l2(rs.row(k), row_bytes);
        pprev = k;
      }
      cp_async_commit();  // one group per pair (empty past the limit)
      ++pf;
    };
#pragma unroll
    for (int j = 0; j < R; ++j) produce();

    unsigned cur = cur0;
    int mode;
    if (start > 0 && prev == cur) {
      mode = (back2 == cur || fwd1 == cur) ? 1 : 0;
    } else {
      ++nseg;
      mode = (has2 && fwd2 == cur) ? 3 : 2;
    }
    RowBuf<OPT, NV> rb;
    if (mode == 2 && cur < nrows) rb.load(rs.row(cur), dim, gl, G);

    double acc[NV][4];
#pragma unroll
    for (int q = 0; q < NV; ++q)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[q][e] = 0.0;

    // the optimizer step on row `key` with the gradient in acc (rb holds the row)
    auto update = [&](unsigned key) {
      double sq = 0.0;
      if (OPT == 3) {
#pragma unroll
        for (int q = 0; q < NV; ++q)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const double g = (double)(float)acc[q][e];
            sq += g * g;
          }
#pragma unroll
        for (int o = 1; o < G; o <<= 1) sq += __shfl_xor_sync(gmask, sq, o, G);
      }
      rb.step_store(rs.row(key), dim, gl, G, acc, oa, sq);
    };
    auto add_owner = [&](unsigned oc) {  // for the combine kernels
      const unsigned slot = atomicAdd(owner_ctr, 1u);
      if (slot < (unsigned)nchunks) owners[slot] = oc;
      else latch(st, kErrInternal);
    };
    // Arrival of a long segment's piece (its partial written), as in
    // bwd_segw_kernel: the owner adds 1 + c + bias, the piece where the
    // segment ends 1 + bias - c, any other piece 1; the group whose addition
    // completes 1 + 2 bias adds the pieces up in chunk order and steps the row
    // (or, past max_pieces, hands the segment to the combine kernels).  A
    // chunk has at most two such pieces, its first (mode 1) and its last
    // (mode 3); their arrivals wait until the chunk's pairs are done, which
    // keeps this code out of the loop over pairs.
    auto arrive = [&](unsigned key, int pmode, bool is_end) {
      unsigned slot = ~0u, fin = 0u;
      if (gl == 0) {
        slot = run_slot(rt, key, st);
        if (slot != ~0u) {
          if (pmode == 3) *(volatile unsigned*)(rt.c0 + slot) = (unsigned)c;
          if (is_end) *(volatile unsigned*)(rt.c1 + slot) = (unsigned)c;
        }
      }
      __threadfence();  // this lane's partial (and the chunk index) before the arrival
      __syncwarp(gmask);
      if (gl == 0 && slot != ~0u) {
        unsigned add = 1u;
        if (pmode == 3) add += (unsigned)c + kRunBias;
        if (is_end) add += kRunBias - (unsigned)c;
        const unsigned old = atomicAdd(rt.ctr + slot, add);
        fin = old + add == 1u + 2u * kRunBias ? 1u : 0u;
      }
      fin = __shfl_sync(gmask, fin, 0, G);
      if (!fin) return;
      slot = __shfl_sync(gmask, slot, 0, G);
      __threadfence();
      const unsigned f0 = *(volatile unsigned*)(rt.c0 + slot);
      const unsigned f1 = *(volatile unsigned*)(rt.c1 + slot);
      if (f1 < f0 || f1 >= (unsigned)nchunks) {
        if (gl == 0) latch(st, kErrInternal);
      } else if (f1 - f0 + 1u <= rt.max_pieces) {
        // the first chunk's tail partial, then each later chunk's head
        // partial, added in chunk order (PF pieces in flight)
        constexpr int PF = NV >= 2 ? (OPT == 1 ? 4 : 2) : 4;  // (registers: no spills)
        const unsigned np = f1 - f0 + 1u;
#pragma unroll
        for (int q = 0; q < NV; ++q)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[q][e] = 0.0;
        for (unsigned k0 = 0; k0 < np; k0 += PF) {
          double v[PF][NV][4];
#pragma unroll
          for (int u = 0; u < PF; ++u) {
            const unsigned k = k0 + (unsigned)u;
            const double* src = k == 0 ? part_tail + (long long)f0 * pstride
                                       : part_head + (long long)(f0 + k) * pstride;
#pragma unroll
            for (int q = 0; q < NV; ++q)
#pragma unroll
              for (int e = 0; e < 4; e += 2) {
                const double2 x = k < np ? __ldcg(reinterpret_cast<const double2*>(src + (q * G + gl) * 4 + e))
                                         : make_double2(0.0, 0.0);
                v[u][q][e] = x.x;
                v[u][q][e + 1] = x.y;
              }
          }
#pragma unroll
          for (int u = 0; u < PF; ++u)
            if (k0 + (unsigned)u < np)
#pragma unroll
              for (int q = 0; q < NV; ++q)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[q][e] += v[u][q][e];
        }
        rb.load(rs.row(key), dim, gl, G);
        update(key);
      } else if (gl == 0) {
        add_owner(f0);
      }
    };
    unsigned pend1 = ~0u, pend3 = ~0u;  // rows of the chunk's long pieces awaiting arrival
    bool pend1_end = false;
    // ended: the segment's last pair is in this piece
    auto close_piece = [&](bool ended) {
      if (mode == 1 || mode == 3) {
        double* o = (mode == 1 ? part_head : part_tail) + (long long)c * pstride;
#pragma unroll
        for (int q = 0; q < NV; ++q)
#pragma unroll
          for (int e = 0; e < 4; ++e) o[(q * G + gl) * 4 + e] = acc[q][e];
        if (rt.key != nullptr && cur < nrows) {
          if (mode == 1) {
            pend1 = cur;
            pend1_end = ended;
          } else {
            pend3 = cur;
          }
        } else if (mode == 3 && gl == 0) {  // for the combine; at most one per chunk for sorted pairs
          add_owner((unsigned)c);
        }
      } else if (mode == 2 && cur < nrows) {
        update(cur);
      }
#pragma unroll
      for (int q = 0; q < NV; ++q)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[q][e] = 0.0;
    };

    // ---- consumer: pairs in order
    int cws = start - G;
    unsigned ck = 0u;
    double cm = 0.0;  // EXT: the factor of pair cws + gl
    bool done = false;
    for (int i = start; i < n32; ++i) {
      if (i >= cws + G) {
        cws = i;
        ck = i + gl < n32 ? __ldg(skey + i + gl) : 0u;
        if (EXT) cm = i + gl < n32 ? __ldg(mult + __ldg(sval + i + gl)) : 0.0;
      }
      const unsigned kt = __shfl_sync(gmask, ck, i - cws, G);
      if (kt != cur) {
        close_piece(true);
        if (i >= end) {
          done = true;
          break;
        }
        cur = kt;
        ++nseg;
        mode = (has2 && fwd2 == cur) ? 3 : 2;
        if (mode == 2 && cur < nrows) rb.load(rs.row(cur), dim, gl, G);
      } else if (i == end && mode != 2) {
        close_piece(false);  // a long piece stops at the chunk end
        done = true;
        break;
      }
      cp_async_wait<R - 1>();  // pair i's columns have landed (this lane's own copy)
      const float4* slot = ring + ((i - start) % R) * NV * G;
      const double f = EXT ? __shfl_sync(gmask, cm, i - cws, G) : 1.0;
      if (mode != 0) {
#pragma unroll
        for (int q = 0; q < NV; ++q) {
          const float4 x = slot[q * G + gl];
          if (EXT) {
            acc[q][0] = ext_add(acc[q][0], x.x, f, mean);
            acc[q][1] = ext_add(acc[q][1], x.y, f, mean);
            acc[q][2] = ext_add(acc[q][2], x.z, f, mean);
            acc[q][3] = ext_add(acc[q][3], x.w, f, mean);
          } else {
            acc[q][0] += (double)x.x;
            acc[q][1] += (double)x.y;
            acc[q][2] += (double)x.z;
            acc[q][3] += (double)x.w;
          }
        }
      }
      produce();  // refill the slot just read with pair i + R
    }
    if (!done) close_piece(true);  // reached the end of the array with a piece open
    cp_async_wait_all();  // the ring is reused by the next chunk
    if (pend1 != ~0u) arrive(pend1, 1, pend1_end);
    if (pend3 != ~0u) arrive(pend3, 3, false);
    if (gl == 0) {
      if (cur >= nrows && nseg) --nseg;  // the missing-key run is not a row
      nseg_total += nseg;
    }
  }
  if (gl == 0 && nseg_total) atomicAdd(&st->sum_unique, (unsigned long long)nseg_total);
}

// ---------------------------------------------------------------------------
// Warp-per-chunk segment reduce: the same chunk ownership rules as
// bwd_seg_kernel, but one whole warp walks a chunk's pairs, each lane holding
// CPL consecutive columns of every row.  The chunk's keys (and those of the
// next chunk, for an owned segment that runs past the chunk end) are loaded
// once; run heads become four 32-bit masks, so finding a run's end, its
// ownership and the pair range to stream are warp-uniform scalar steps and
// no lane waits on another lane's control path; the runs are listed once in
// shared memory.  Gradient rows are staged a batch of pairs at a time into
// this warp's two shared-memory buffers by cp.async.bulk (one copy per row,
// issued by the lane of that pair; completion on the buffer's mbarrier, waits
// bounded) and added in fp64 in sorted order; the table row of an owned run is
// loaded into registers one run ahead and written once when the run closes.
// ---------------------------------------------------------------------------
// Pairs per staged batch (two batches per warp in flight or being read): 8 KB
// of rows per warp at every width.
__host__ __device__ constexpr int segw_batch(int cpl) {
  return cpl <= 2 ? 16 : (cpl == 4 ? DHS_SEGW_BATCH4 : 32 / cpl);
}
__host__ __device__ constexpr size_t segw_smem_bytes(int cpl) {
  return (size_t)8 * 2 * segw_batch(cpl) * 32 * cpl * sizeof(float);
}

__device__ __forceinline__ void mbar_init(unsigned bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_arrive(unsigned bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// Waits (bounded) until the phase of the given parity has completed.
constexpr unsigned kMbarSpins = 1u << 22;
__device__ __forceinline__ bool mbar_wait(unsigned bar, unsigned parity) {
  for (unsigned i = 0; i < kMbarSpins; ++i) {
    unsigned done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}
// One row (bytes a multiple of 16, both addresses 16-byte aligned) from
// global into shared memory; completion is counted on the mbarrier.  The L2
// policy marks rows read once as first to evict, so that they do not push out
// the rows and keys the kernel reads again.
__device__ __forceinline__ void bulk_g2s(unsigned dst, const void* src, unsigned bytes, unsigned bar,
                                         unsigned long long policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}
__device__ __forceinline__ unsigned long long l2_policy(bool evict_first) {
  unsigned long long p;
  if (evict_first)
    asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  else
    asm("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// CPL columns of a row at p (p + col0 aligned to the vector width) into v and
// back; columns at or past dim are neither read nor written.
template <int CPL>
__device__ __forceinline__ void segw_ld(float (&v)[CPL], const float* p, int col0, int dim) {
  if constexpr (CPL == 1) {
    v[0] = p[col0];
  } else if constexpr (CPL == 2) {
    const float2 x = *reinterpret_cast<const float2*>(p + col0);
    v[0] = x.x;
    v[1] = x.y;
  } else {
#pragma unroll
    for (int k = 0; k < CPL / 4; ++k) {
      if (col0 + 4 * k < dim) {
        const float4 x = *reinterpret_cast<const float4*>(p + col0 + 4 * k);
        v[4 * k] = x.x;
        v[4 * k + 1] = x.y;
        v[4 * k + 2] = x.z;
        v[4 * k + 3] = x.w;
      }
    }
  }
}
// CPL consecutive bf16 weights at element col0 of the row at p, widened to
// fp32 and back (rounded to nearest even); as segw_ld / segw_st, columns at or
// past dim are neither read nor written (dim is a multiple of 8).
template <int CPL>
__device__ __forceinline__ void segw_ld_bf(float (&v)[CPL], const float* p, int col0, int dim) {
  const unsigned short* h = reinterpret_cast<const unsigned short*>(p) + col0;
  if constexpr (CPL == 1) {
    v[0] = __uint_as_float((unsigned)h[0] << 16);
  } else if constexpr (CPL == 2) {
    const unsigned u = *reinterpret_cast<const unsigned*>(h);
    v[0] = bf16_lo(u);
    v[1] = bf16_hi(u);
  } else if constexpr (CPL == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(h);
    v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
  } else {
#pragma unroll
    for (int k = 0; k < CPL / 8; ++k) {
      if (col0 + 8 * k < dim) {
        const uint4 u = *reinterpret_cast<const uint4*>(h + 8 * k);
        v[8 * k + 0] = bf16_lo(u.x); v[8 * k + 1] = bf16_hi(u.x);
        v[8 * k + 2] = bf16_lo(u.y); v[8 * k + 3] = bf16_hi(u.y);
        v[8 * k + 4] = bf16_lo(u.z); v[8 * k + 5] = bf16_hi(u.z);
        v[8 * k + 6] = bf16_lo(u.w); v[8 * k + 7] = bf16_hi(u.w);
      }
    }
  }
}
template <int CPL>
__device__ __forceinline__ void segw_st_bf(float* p, const float (&v)[CPL], int col0, int dim) {
  unsigned short* h = reinterpret_cast<unsigned short*>(p) + col0;
  if constexpr (CPL == 1) {
    *reinterpret_cast<__nv_bfloat16*>(h) = __float2bfloat16_rn(v[0]);
  } else if constexpr (CPL == 2) {
    *reinterpret_cast<unsigned*>(h) = pack_bf16x2(v[0], v[1]);
  } else if constexpr (CPL == 4) {
    *reinterpret_cast<uint2*>(h) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
  } else {
#pragma unroll
    for (int k = 0; k < CPL / 8; ++k)
      if (col0 + 8 * k < dim)
        *reinterpret_cast<uint4*>(h + 8 * k) =
            make_uint4(pack_bf16x2(v[8 * k], v[8 * k + 1]), pack_bf16x2(v[8 * k + 2], v[8 * k + 3]),
                       pack_bf16x2(v[8 * k + 4], v[8 * k + 5]), pack_bf16x2(v[8 * k + 6], v[8 * k + 7]));
  }
}

template <int CPL>
__device__ __forceinline__ void segw_st(float* p, const float (&v)[CPL], int col0, int dim) {
  if constexpr (CPL == 1) {
    p[col0] = v[0];
  } else if constexpr (CPL == 2) {
    *reinterpret_cast<float2*>(p + col0) = make_float2(v[0], v[1]);
  } else {
#pragma unroll
    for (int k = 0; k < CPL / 4; ++k)
      if (col0 + 4 * k < dim)
        *reinterpret_cast<float4*>(p + col0 + 4 * k) =
            make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
  }
}

// EXT (extended pooling): sort values are positions; the pair's bag is
// bagpos[position] and its gradient row is multiplied by mult[position] (a
// per-sample weight) or, with mean, divided by it (the bag's length), both
// gathered once per chunk.
// BF: the table's weights are bf16 (state fp32): loaded widened, updated in
// fp32, stored rounded to nearest even.
template <int CPL, int OPT, bool EXT, bool BF>
__global__ void __launch_bounds__(256, CPL <= 4 ? DHS_SEGW_MINB : 1)
bwd_segw_kernel(const unsigned* __restrict__ skey, const unsigned* __restrict__ sval, long long n,
                const float* __restrict__ grad, long long n_bags, int dim, RowSpace rs, OptArgs oa,
                double* __restrict__ part_head, double* __restrict__ part_tail, int pstride, int C,
                unsigned* __restrict__ chunk_ctr, unsigned* __restrict__ owners,
                unsigned* __restrict__ owner_ctr, DevState* st, bool grad_once,
                const unsigned* __restrict__ bagpos, const double* __restrict__ mult, bool mean,
                RunTable rt) {
  pdl_enter();
  constexpr int B = segw_batch(CPL);
  constexpr int PITCH = 32 * CPL;  // floats per staged row
  constexpr int NS = seg_state_arrays(OPT);
  constexpr unsigned FULL = 0xffffffffu;
  extern __shared__ __align__(128) float segw_smem[];
  __shared__ __align__(8) unsigned long long segw_bar[8][2];
  __shared__ uint2 segw_runs[8][130];  // per warp: the stream's runs {key, start | mode << 16}
  __shared__ double segw_mult[EXT ? 8 : 1][EXT ? 128 : 1];  // per warp: each pair's factor
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  const int col0 = lane * CPL;
  const bool lane_on = col0 < dim;
  float* wbuf = segw_smem + (size_t)wid * 2 * B * PITCH;  // this warp's two batches of rows
  const unsigned wbuf_s = (unsigned)__cvta_generic_to_shared(wbuf);
  const unsigned bar_s = (unsigned)__cvta_generic_to_shared(&segw_bar[wid][0]);
  if (lane == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_s + 8, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  unsigned parity = 0;  // bit b: parity of the next phase of batch buffer b
  bool broken = false;
  const unsigned long long grad_policy = l2_policy(grad_once);
  // positions and bags fit in 31 bits (the host rejects larger calls); C <= 64
  const int n32 = (int)n;
  const unsigned nb32 = (unsigned)n_bags;
  const int nchunks = (n32 + C - 1) / C;
  const unsigned nrows = (unsigned)min(st->row_count, 0xffffffffull);
  unsigned nseg_total = 0;

  for (;;) {
    int c = 0;
    if (lane == 0) c = (int)atomicAdd(chunk_ctr, 1u);
    c = __shfl_sync(FULL, c, 0);
    if (c >= nchunks) break;
    // chunks are handed out from the end of the sorted pairs: rows sort in
    // the order they were created, so the high rows (keys seen recently, in
    // short segments, a row update every few pairs: the slow chunks) go
    // first and the chunks inside long segments of old hot rows last
    if (DHS_SEGW_REVERSE) c = nchunks - 1 - c;
    const int start = c * C;
    const int end = min(n32, start + C);
    const int limit = min(n32, end + C);  // an owned run ends before chunk c + 2
    const int lim = limit - start, cend = end - start;  // relative to start

    // keys and bags of [start, limit), 32 per word
    unsigned kw[4], vw[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int p = start + 32 * w + lane;
      const bool in = p < limit;
      kw[w] = in ? __ldg(skey + p) : ~0u;
      vw[w] = in ? __ldg(sval + p) : 0u;
    }
    if constexpr (EXT) {
      // positions -> bags, and each pair's factor into this warp's list (the
      // previous chunk's readers passed the warp-wide shuffle at the loop top)
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const bool in = start + 32 * w + lane < limit;
        const unsigned pos = vw[w];
        segw_mult[wid][32 * w + lane] = in ? __ldg(mult + pos) : 0.0;
        vw[w] = in ? __ldg(bagpos + pos) : 0u;
      }
      __syncwarp();
    }
    const unsigned prev = start > 0 ? __ldg(skey + start - 1) : ~0u;
    const unsigned back2 = c >= 2 ? __ldg(skey + (c - 1) * C - 1) : ~0u;
    const unsigned fwd1 = end < n32 ? __ldg(skey + end) : ~0u;
    const bool has2 = (c + 2) * C < n32;
    const unsigned fwd2 = has2 ? __ldg(skey + (c + 2) * C) : ~0u;
    // run heads: bit q of word q / 32 set when position start + q starts a run
    unsigned hm[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      unsigned before = __shfl_up_sync(FULL, kw[w], 1);
      const unsigned carry = w == 0 ? prev : __shfl_sync(FULL, kw[w == 0 ? 0 : w - 1], 31);
      if (lane == 0) before = carry;
      hm[w] = __ballot_sync(FULL, 32 * w + lane < lim && kw[w] != before);
    }
    auto word = [&](const unsigned (&a)[4], int q) -> unsigned {
      return q < 32 ? a[0] : (q < 64 ? a[1] : (q < 96 ? a[2] : a[3]));
    };
    auto key_at = [&](int q) -> unsigned { return __shfl_sync(FULL, word(kw, q), q & 31); };
    // first head after relative position q, or lim
    auto next_head = [&](int q) -> int {
      int r = q + 1;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        if (r < 32 * (w + 1) && r < lim) {
          unsigned m = w == 0 ? hm[0] : (w == 1 ? hm[1] : (w == 2 ? hm[2] : hm[3]));
          const int lo = r - 32 * w;
          if (lo > 0) m &= 0xffffffffu << lo;
          if (m) return 32 * w + __ffs(m) - 1;
          r = 32 * (w + 1);
        }
      }
      return lim;
    };
    // last head at or before relative position q (0 when the first run covers it)
    auto last_head = [&](int q) -> int {
#pragma unroll
      for (int w = 3; w >= 0; --w) {
        if (32 * w <= q) {
          unsigned m = w == 0 ? hm[0] : (w == 1 ? hm[1] : (w == 2 ? hm[2] : hm[3]));
          const int hi = q - 32 * w;
          if (hi < 31) m &= (2u << hi) - 1u;
          if (m) return 32 * w + 31 - __clz(m);
        }
      }
      return 0;
    };

    // ownership: the first run continues one from the previous chunk unless a
    // head sits at position 0; runs that reach chunk c + 2 are long
    const unsigned k0 = key_at(0);
    const bool first_here = hm[0] & 1u;
    const int mode_first = first_here ? ((has2 && fwd2 == k0) ? 3 : 2)
                                      : ((back2 == k0 || fwd1 == k0) ? 1 : 0);
    const int s0 = mode_first == 0 ? next_head(0) : 0;
    const int hl = last_head(cend - 1);
    const unsigned kl = key_at(cend - 1);
    const int mode_last = hl == 0 ? mode_first : ((has2 && fwd2 == kl) ? 3 : 2);
    const int stop = mode_last == 2 ? next_head(cend - 1) : (mode_last == 0 ? s0 : cend);

    // distinct rows started in this chunk
    {
      unsigned cnt = 0;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const bool head = (hm[w] >> lane) & 1u;
        cnt += __popc(__ballot_sync(FULL, head && 32 * w + lane < cend && kw[w] < nrows));
      }
      nseg_total += cnt;
    }
    if (s0 >= stop) continue;

    // the stream's runs: entry 0 starts at s0, then one entry per head in
    // (s0, stop), then a sentinel at stop; owned rows are prefetched into L2
    uint2* runs = segw_runs[wid];
    int nruns;
    {
      const unsigned ks0 = key_at(s0);
      unsigned base = 1;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int q = 32 * w + lane;
        const bool h = ((hm[w] >> lane) & 1u) && q > s0 && q < stop;
        const unsigned m = __ballot_sync(FULL, h);
        if (h) {
          const unsigned k = kw[w];
          const unsigned md = (has2 && fwd2 == k) ? 3u : 2u;
          runs[base + __popc(m & lanemask_lt())] = make_uint2(k, (unsigned)q | (md << 16));
          if (md == 2u && k < nrows) prefetch_l2(rs.row(k), (unsigned)rs.stride * 4u);
        }
        base += __popc(m);
      }
      nruns = (int)base;
      if (lane == 0) {
        const unsigned md = s0 == 0 ? (unsigned)mode_first : ((has2 && fwd2 == ks0) ? 3u : 2u);
        runs[0] = make_uint2(ks0, (unsigned)s0 | (md << 16));
        runs[nruns] = make_uint2(0u, (unsigned)stop);
        if (md == 2u && ks0 < nrows) prefetch_l2(rs.row(ks0), (unsigned)rs.stride * 4u);
      }
      __syncwarp();
    }

    // ---- producer: the gradient rows of stream batch j (pairs s0 + j B ...)
    // into buffer j & 1, one bulk copy per row issued by the lane of that
    // pair.  A pair whose key has no row or whose bag is out of range is not
    // copied and not added.
#pragma unroll
    for (int w = 0; w < 4; ++w) vw[w] = (kw[w] < nrows && vw[w] < nb32) ? vw[w] : ~0u;
    const int nbat = (stop - s0 + B - 1) / B;
    const unsigned row_bytes = (unsigned)dim * 4u;
    auto issue = [&](int j) -> unsigned {
      const int q0 = s0 + j * B;
      const int q = q0 + lane;
      const int w0 = q0 >> 5;
      const unsigned a0 = __shfl_sync(FULL, word(vw, 32 * w0), q & 31);
      const unsigned a1 = __shfl_sync(FULL, word(vw, min(32 * w0 + 32, 127)), q & 31);
      const unsigned bg = (q >> 5) == w0 ? a0 : a1;
      const bool valid = lane < B && q < stop && bg != ~0u;
      const unsigned vmask = __ballot_sync(FULL, valid);
      const unsigned bar = bar_s + 8u * (j & 1);
      // the buffer's previous rows were read by this warp's generic loads
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      if (lane == 0) mbar_expect_arrive(bar, (unsigned)__popc(vmask) * row_bytes);
      __syncwarp();
      if (valid)
        bulk_g2s(wbuf_s + (unsigned)(((j & 1) * B + lane) * PITCH) * 4u, grad + (size_t)bg * dim, row_bytes, bar,
                 grad_policy);
      return vmask;
    };

    // ---- consumer
    double acc[CPL];
#pragma unroll
    for (int e = 0; e < CPL; ++e) acc[e] = 0.0;
    float rw[CPL];
    float rst[NS > 0 ? NS : 1][CPL];
    float racc = 0.f;
    unsigned kcur = 0;
    int mode = 0, run_end = 0;
    unsigned rslot = 0;  // lane 0: arrival entry of the current piece
    // the row of an owned run, loaded into the "next" registers one run ahead
    float nw[CPL];
    float nst[NS > 0 ? NS : 1][CPL];
    float nra = 0.f;
    const int wfl = rs.wfl;  // the state starts wfl floats into the row
    auto fetch = [&](uint2 e) {
      if ((e.y >> 16) == 2u && e.x < nrows) {
        const float* row = rs.row(e.x);
        if (lane_on) {
          if constexpr (BF)
            segw_ld_bf<CPL>(nw, row, col0, dim);
          else
            segw_ld<CPL>(nw, row, col0, dim);
#pragma unroll
          for (int k = 0; k < NS; ++k) segw_ld<CPL>(nst[k], row + wfl + k * dim, col0, dim);
        }
        if (OPT == 3) nra = row[wfl];
      }
    };
    // the optimizer step on the row of kcur with the gradient in acc and the
    // row's values in rw / rst / racc
    auto update_row = [&](float* row) {
      float den = 0.f, Gn = 0.f;
      if (OPT == 3) {
        double sq = 0.0;
#pragma unroll
        for (int e = 0; e < CPL; ++e) {
          if (lane_on && col0 + e < dim) {
            const double g = (double)(float)acc[e];
            sq += g * g;
          }
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) sq += __shfl_xor_sync(FULL, sq, o);
        Gn = __fadd_rn(racc, (float)(sq / (double)dim));
        den = __fadd_rn(__fsqrt_rn(Gn), oa.eps);
      }
      if (lane_on) {
#pragma unroll
        for (int e = 0; e < CPL; ++e) {
          const float g = (float)acc[e];
          if (OPT == 0) {
            rw[e] = sgd_w(rw[e], g, oa.lr);
          } else if (OPT == 1) {
            adagrad_step(rw[e], rst[0][e], g, oa.lr, oa.eps);
          } else if (OPT == 2) {
            adam_step(rw[e], rst[0][e], rst[NS - 1][e], g, oa);
          } else {
            rw[e] = __fsub_rn(rw[e], __fdiv_rn(__fmul_rn(oa.lr, g), den));
          }
        }
        if constexpr (BF)
          segw_st_bf<CPL>(row, rw, col0, dim);
        else
          segw_st<CPL>(row, rw, col0, dim);
#pragma unroll
        for (int k = 0; k < NS; ++k) segw_st<CPL>(row + wfl + k * dim, rst[k], col0, dim);
      }
      if (OPT == 3 && lane == 0) row[wfl] = Gn;
    };
    // the warp that brings the last piece of a long segment finishes it: the
    // pieces (the first chunk's tail partial, then each later chunk's head
    // partial) added in chunk order into acc, then the optimizer step
    auto finish_long = [&](unsigned f0, unsigned np) {
      constexpr int FB = CPL <= 2 ? 8 : (CPL == 4 ? 4 : (CPL == 8 ? 2 : 1));  // pieces in flight
#pragma unroll
      for (int e = 0; e < CPL; ++e) acc[e] = 0.0;
      if (lane_on) {
        for (unsigned k0 = 0; k0 < np; k0 += FB) {
          double v[FB][CPL];
#pragma unroll
          for (int i = 0; i < FB; ++i) {
            const unsigned k = k0 + (unsigned)i;
            const double* src =
                (k == 0 ? part_tail + (long long)f0 * pstride : part_head + (long long)(f0 + k) * pstride) + col0;
            if constexpr (CPL == 1) {
              v[i][0] = k < np ? __ldcg(src) : 0.0;
            } else {
#pragma unroll
              for (int e = 0; e < CPL; e += 2) {
                const double2 x = k < np && col0 + e < dim ? __ldcg(reinterpret_cast<const double2*>(src + e))
                                                           : make_double2(0.0, 0.0);
                v[i][e] = x.x;
                v[i][e + 1] = x.y;
              }
            }
          }
#pragma unroll
          for (int i = 0; i < FB; ++i)
            if (k0 + (unsigned)i < np)
#pragma unroll
              for (int e = 0; e < CPL; ++e) acc[e] += v[i][e];
        }
      }
      float* row = rs.row(kcur);
      if (lane_on) {
        if constexpr (BF)
          segw_ld_bf<CPL>(rw, row, col0, dim);
        else
          segw_ld<CPL>(rw, row, col0, dim);
#pragma unroll
        for (int k = 0; k < NS; ++k) segw_ld<CPL>(rst[k], row + wfl + k * dim, col0, dim);
      }
      if (OPT == 3) racc = row[wfl];
      update_row(row);
    };
    auto add_owner = [&](unsigned oc) {  // for the combine kernels
      const unsigned slot = atomicAdd(owner_ctr, 1u);
      if (slot < (unsigned)nchunks) owners[slot] = oc;
      else latch(st, kErrInternal);
    };
    auto close = [&]() {
      if (mode == 1 || mode == 3) {
        double* o = (mode == 1 ? part_head : part_tail) + (long long)c * pstride + col0;
        if (lane_on) {
#pragma unroll
          for (int e = 0; e < CPL; ++e)
            if (col0 + e < dim) o[e] = acc[e];
        }
        if (rt.key != nullptr && kcur < nrows) {
          // arrival: the owner adds 1 + c + bias, the chunk where the segment
          // ends 1 + bias - c, every other piece 1; the sum reaches
          // 1 + 2 bias exactly when all c1 - c0 + 1 pieces have arrived, in
          // whatever order (no partial sum can reach it: chunks < 2^26)
          const unsigned slot0 = rslot;
          const bool is_end = mode == 1 && (run_end < cend || fwd1 != kcur);
          if (lane == 0 && slot0 != ~0u) {
            if (mode == 3) *(volatile unsigned*)(rt.c0 + slot0) = (unsigned)c;
            if (is_end) *(volatile unsigned*)(rt.c1 + slot0) = (unsigned)c;
          }
          __threadfence();  // this lane's partial (and lane 0's chunk index) before the arrival
          __syncwarp();
          unsigned fin = 0, slot = slot0;
          if (lane == 0 && slot0 != ~0u) {
            unsigned add = 1u;
            if (mode == 3) add += (unsigned)c + kRunBias;
            if (is_end) add += kRunBias - (unsigned)c;
            const unsigned old = atomicAdd(rt.ctr + slot0, add);
            fin = old + add == 1u + 2u * kRunBias ? 1u : 0u;
          }
          fin = __shfl_sync(FULL, fin, 0);
          if (fin) {
            slot = __shfl_sync(FULL, slot, 0);
            __threadfence();
            const unsigned f0 = *(volatile unsigned*)(rt.c0 + slot);
            const unsigned f1 = *(volatile unsigned*)(rt.c1 + slot);
            if (f1 < f0 || f1 >= (unsigned)nchunks) {
              if (lane == 0) latch(st, kErrInternal);
            } else if (f1 - f0 + 1u <= rt.max_pieces) {
              finish_long(f0, f1 - f0 + 1u);
            } else if (lane == 0) {
              add_owner(f0);
            }
          }
        } else if (mode == 3 && lane == 0) {  // at most one per chunk for sorted pairs
          add_owner((unsigned)c);
        }
      } else if (mode == 2 && kcur < nrows) {
        update_row(rs.row(kcur));
      }
#pragma unroll
      for (int e = 0; e < CPL; ++e) acc[e] = 0.0;
    };

    uint2 ecur = runs[0];
    fetch(ecur);
    unsigned vm[2];
    vm[0] = issue(0);
    vm[1] = nbat > 1 ? issue(1) : 0u;
    // batch j holds stream pairs [q0, qbe); runs are the outer loop, the pairs
    // of a run inside one batch a tight inner loop
    int j = 0, q0 = s0, qbe = min(s0 + B, stop), q = s0;
    unsigned vmask = vm[0];
    const float* rows = wbuf + col0;
    if (!mbar_wait(bar_s, parity & 1u)) {
      latch(st, kErrInternal);  // a row copy never completed
      broken = true;
      break;
    }
    parity ^= 1u;
    for (int r = 0; r < nruns && !broken; ++r) {
      kcur = ecur.x;
      mode = (int)(ecur.y >> 16);
      const uint2 enext = runs[r + 1];
      run_end = (int)(enext.y & 0xffffu);
      if (mode != 2) run_end = min(run_end, cend);  // a long piece stops at the chunk end
      // a piece of a long segment finds its arrival entry now, so that the
      // lookup's latency passes while the piece is summed
      if ((mode == 1 || mode == 3) && lane == 0 && rt.key != nullptr && kcur < nrows)
        rslot = run_slot(rt, kcur, st);
#pragma unroll
      for (int e = 0; e < CPL; ++e) rw[e] = nw[e];
#pragma unroll
      for (int k = 0; k < NS; ++k)
#pragma unroll
        for (int e = 0; e < CPL; ++e) rst[k][e] = nst[k][e];
      racc = nra;
      if (r + 1 < nruns) fetch(enext);  // in flight while this run is summed
      ecur = enext;
      while (q < run_end) {
        if (q == qbe) {
          // next batch: refill the buffer just finished, wait for the other
          __syncwarp();  // every lane has read this buffer
          if (j + 2 < nbat) {
            const unsigned m = issue(j + 2);
            if (j & 1) vm[1] = m; else vm[0] = m;
          }
          ++j;
          const int bsel = j & 1;
          if (!mbar_wait(bar_s + 8u * bsel, (parity >> bsel) & 1u)) {
            latch(st, kErrInternal);
            broken = true;
            break;
          }
          parity ^= 1u << bsel;
          vmask = bsel ? vm[1] : vm[0];
          rows = wbuf + bsel * B * PITCH + col0;
          q0 = s0 + j * B;
          qbe = min(q0 + B, stop);
        }
        const int qe = min(run_end, qbe);
        if (lane_on) {
          for (; q < qe; ++q) {
            const int i = q - q0;
            if ((vmask >> i) & 1u) {
              float x[CPL];
#pragma unroll
              for (int e = 0; e < CPL; ++e) x[e] = 0.f;
              segw_ld<CPL>(x, rows + i * PITCH, 0, dim - col0);
              if constexpr (EXT) {
                const double f = segw_mult[wid][q];
#pragma unroll
                for (int e = 0; e < CPL; ++e) acc[e] = ext_add(acc[e], x[e], f, mean);
              } else {
#pragma unroll
                for (int e = 0; e < CPL; ++e) acc[e] += (double)x[e];
              }
            }
          }
        } else {
          q = qe;
        }
      }
      if (broken) break;
      close();
    }
    if (broken) break;
  }
  if (broken) {
    // let the other buffer's copies (if any) land before the block exits
    for (int b = 0; b < 2; ++b) (void)mbar_wait(bar_s + 8u * b, (parity >> b) & 1u);
  }
  if (lane == 0 && nseg_total) atomicAdd(&st->sum_unique, (unsigned long long)nseg_total);
}

#ifndef DHS_TEMPLATES_ONLY
// Long segments (the owner chunks the segment kernel listed) are finished in
// two launches.  Plan: one warp per owner finds the chunk holding the
// segment's last pair (the first pairs of the run's chunks all carry the key;
// keys are sorted, so a 32-way search over chunk starts finds the last one),
// cuts the run's pieces (the owner's starting partial, then one head piece
// per following chunk) into batches of about sqrt(pieces) each and takes
// batch ids (and, for runs of more than one batch, fp64 slots) from counters.
// Combine: one block per batch adds its pieces in fp64; a one-batch run
// updates its row directly, otherwise the batch stores its sum in its slot and
// the last of the run's batches to finish (an atomic ticket; no block waits)
// adds the slots in batch order and applies the optimizer once.  Every sum is
// taken in an order fixed by the run alone.  With batches of about sqrt(pieces)
// both the batch sums and the final sum over the slots are short chains of
// loads, for a run of a few hundred pieces as for one of tens of thousands.
constexpr int kCombineThreads = 256;
constexpr int kCombineMinPieces = 16;

// Pieces per batch of a run of npieces pieces: the smallest power of two of
// at least kCombineMinPieces whose square reaches npieces.
__host__ __device__ inline unsigned combine_batch_pieces(long long npieces) {
  unsigned p = kCombineMinPieces;
  while ((long long)p * p < npieces) p <<= 1;
  return p;
}

// Runs of at most this many pieces are finished by the plan kernel's warp.
constexpr int kWarpFinishPieces = 16;

// One warp finishes a run of npieces pieces: piece 0 at first, piece k >= 1
// at rest + (k - 1) * pstride; lane l owns columns l + 32 i (dim <= 512).
__device__ __forceinline__ void finish_run_warp(float* row, int dim, int wfl, const OptArgs& oa,
                                                const double* first, const double* rest, int pstride,
                                                long long npieces, int lane) {
  constexpr int kCols = 16;  // columns per lane at dim 512
  float g[kCols];
  double sq = 0.0;
#pragma unroll
  for (int i = 0; i < kCols; ++i) {
    const int j = lane + 32 * i;
    g[i] = 0.f;
    if (j < dim) {
      // every piece of the column in flight at once, then added in order
      double v[kWarpFinishPieces];
      v[0] = __ldcg(first + j);
#pragma unroll
      for (int k = 1; k < kWarpFinishPieces; ++k) v[k] = k < npieces ? __ldcg(rest + (k - 1) * pstride + j) : 0.0;
      double a = v[0];
#pragma unroll
      for (int k = 1; k < kWarpFinishPieces; ++k)
        if (k < npieces) a += v[k];
      g[i] = (float)a;
      const double gd = (double)g[i];
      sq += gd * gd;
    }
  }
  float den = 0.f, Gn = 0.f;
  if (oa.opt == 3) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    Gn = __fadd_rn(row[wfl], (float)(sq / (double)dim));
    den = __fadd_rn(__fsqrt_rn(Gn), oa.eps);
  }
#pragma unroll
  for (int i = 0; i < kCols; ++i) {
    const int j = lane + 32 * i;
    if (j < dim) update_col(row, dim, wfl, j, g[i], oa, den);
  }
  if (oa.opt == 3 && lane == 0) row[wfl] = Gn;
}

struct CombinePlan {
  unsigned* key;          // [owners] row of the run
  unsigned* kend;         // [owners] chunk holding the last pair
  unsigned* boff;         // [owners] first batch id
  unsigned* sbase;        // [owners] first slot (runs of more than one batch)
  unsigned* ticket;       // [owners] batches finished
  unsigned* ppb;          // [owners] pieces per batch
  unsigned* batch_owner;  // [batch_cap] owner of each batch id
  double* slots;          // [slot_cap][pstride]
  unsigned batch_cap, slot_cap;
  unsigned owner_cap;     // entries of the owner list and of the per-owner arrays
  unsigned* batch_ctr;    // zeroed before the segment kernel
  unsigned* slot_ctr;
};

__global__ void __launch_bounds__(256)
bwd_combine_plan_kernel(const unsigned* __restrict__ skey, long long n, int C,
                        const unsigned* __restrict__ owners, const unsigned* __restrict__ owner_ctr,
                        CombinePlan pl, int dim, RowSpace rs, OptArgs oa,
                        const double* __restrict__ part_head, const double* __restrict__ part_tail,
                        int pstride, DevState* st) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const long long nchunks = (n + C - 1) / C;
  const unsigned long long nrows = st->row_count;
  const unsigned n_own = (unsigned)min((long long)*owner_ctr, nchunks);  // the seg kernel wrote [0, n_own)
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long oi = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); oi < n_own;
       oi += warps) {
    const long long c = owners[oi];
    const unsigned key = skey[(c + 1) * (long long)C - 1];
    long long lo = c + 1, hi = nchunks - 1;  // the last chunk is in [lo, hi]; chunk c + 1 is in the run
    while (lo < hi) {
      const long long stride = (hi - lo + 32) / 32;
      const long long kk = lo + lane * stride;
      const unsigned in_run = __ballot_sync(0xffffffffu, kk <= hi && skey[kk * C] == key);
      // lane 0 (chunk lo) is in the run when the pairs are sorted; counting it
      // in regardless keeps lo >= c + 1 whatever the input
      lo += (long long)(31 - __clz(in_run | 1u)) * stride;
      hi = min(hi, lo + stride - 1);
      if (stride == 1) break;
    }
    const long long npieces = lo - c + 1;
    const unsigned P = combine_batch_pieces(npieces);
    unsigned nb = key < nrows ? (unsigned)((npieces + P - 1) / P) : 0u;
    if (key < nrows && npieces <= kWarpFinishPieces) {
      // a short run is finished here by this warp: lane l sums columns l,
      // l + 32, ... over the pieces in order (piece 0 = the owner's starting
      // partial), then applies the optimizer; no batch is planned for it
      finish_run_warp(rs.row(key), dim, rs.wfl, oa, part_tail + c * (long long)pstride,
                      part_head + (c + 1) * (long long)pstride, pstride, npieces, lane);
      nb = 0;
    }
    unsigned base = 0, sb = 0;
    if (lane == 0) {
      base = atomicAdd(pl.batch_ctr, nb);
      if (nb > 1) sb = atomicAdd(pl.slot_ctr, nb);
      if (base + nb > pl.batch_cap || (nb > 1 && sb + nb > pl.slot_cap)) {
        latch(st, kErrInternal);  // the caps bound every run of sorted input
        base = pl.batch_cap;
      }
      pl.key[oi] = key;
      pl.kend[oi] = (unsigned)lo;
      pl.boff[oi] = base;
      pl.sbase[oi] = sb;
      pl.ticket[oi] = 0u;
      pl.ppb[oi] = P;
    }
    base = __shfl_sync(0xffffffffu, base, 0);
    for (unsigned j = lane; j < nb && base + j < pl.batch_cap; j += 32) pl.batch_owner[base + j] = (unsigned)oi;
  }
}

__global__ void __launch_bounds__(kCombineThreads, 4)
bwd_combine_kernel(const unsigned* __restrict__ skey, int dim, RowSpace rs, OptArgs oa,
                   const double* __restrict__ part_head, const double* __restrict__ part_tail, int C,
                   int pstride, const unsigned* __restrict__ owners,
                   const unsigned* __restrict__ owner_ctr, CombinePlan pl) {
  pdl_enter();
  extern __shared__ double sacc[];  // [slices][dim]
  __shared__ double s_sq;
  __shared__ bool s_last;
  const int T = blockDim.x;
  const int slices = dim >= T ? 1 : T / dim;
  const unsigned nbatch = min(*pl.batch_ctr, pl.batch_cap);
  const unsigned n_own = min(*owner_ctr, pl.owner_cap);  // the count may pass the list after a failed sort
  for (unsigned bid = blockIdx.x; bid < nbatch; bid += gridDim.x) {
    const unsigned oi = pl.batch_owner[bid];
    if (oi >= n_own) continue;  // only after a plan overflow, which the plan reported
    const long long c = owners[oi];
    const unsigned key = pl.key[oi];
    const long long npieces = (long long)pl.kend[oi] - c + 1;
    const unsigned b = bid - pl.boff[oi];
    const unsigned P = pl.ppb[oi];
    const unsigned nb = (unsigned)((npieces + P - 1) / P);
    if (b >= nb) continue;
    // the plan gives no batch to a missing-key run; this thread's column of
    // the row (rows of at most T floats) is loaded while the pieces are summed
    float* const row = rs.row(key);
    const int wfl = rs.wfl;
    const bool bf16 = wfl != dim;
    const bool pre = dim <= T && (int)threadIdx.x < dim;
    float pw = 0.f, ps0 = 0.f, ps1 = 0.f;
    if (pre) {
      pw = load_w(row, threadIdx.x, bf16);
      if (oa.opt == 1 || oa.opt == 2) ps0 = row[wfl + threadIdx.x];
      if (oa.opt == 2) ps1 = row[wfl + dim + threadIdx.x];
    }
    const long long p0 = (long long)b * P;
    const long long p1 = min(npieces, p0 + (long long)P);
    // slice sl adds pieces p0 + sl, p0 + sl + slices, ... (piece 0 = starting partial)
    for (int j0 = 0; j0 < dim; j0 += (slices == 1 ? T : dim)) {
      const int sl = slices == 1 ? 0 : threadIdx.x / dim;
      const int j = slices == 1 ? j0 + threadIdx.x : threadIdx.x % dim;
      if (sl < slices && j < dim) {
        auto piece = [&](long long pc) -> double {
          const double* src = pc == 0 ? part_tail + c * (long long)pstride
                                      : part_head + (c + pc) * (long long)pstride;
          return __ldcg(src + j);
        };
        double a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        long long pc = p0 + sl;
        for (; pc + 7LL * slices < p1; pc += 8LL * slices) {
#pragma unroll
          for (int u = 0; u < 8; ++u) a[u] += piece(pc + (long long)u * slices);
        }
        for (; pc < p1; pc += slices) a[0] += piece(pc);
        sacc[sl * dim + j] = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
      }
      if (slices != 1) break;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < dim && slices > 1; j += T) {
      double a = sacc[j];
      for (int s2 = 1; s2 < slices; ++s2) a += sacc[s2 * dim + j];
      sacc[j] = a;
    }
    __syncthreads();
    if (nb > 1) {
      double* mine = pl.slots + (size_t)(pl.sbase[oi] + b) * pstride;
      for (int j = threadIdx.x; j < dim; j += T) mine[j] = sacc[j];
      __threadfence();
      __syncthreads();
      if (threadIdx.x == 0) s_last = atomicAdd(&pl.ticket[oi], 1u) == nb - 1u;
      __syncthreads();
      if (!s_last) continue;  // uniform across the block
      __threadfence();
      const double* all = pl.slots + (size_t)pl.sbase[oi] * pstride;
      for (int j = threadIdx.x; j < dim; j += T) {
        double a = 0.0;
        for (unsigned k = 0; k < nb; ++k) a += __ldcg(all + (size_t)k * pstride + j);
        sacc[j] = a;
      }
      __syncthreads();
    }
    float den = 0.f;
    if (oa.opt == 3) {
      if (threadIdx.x == 0) {
        double sq = 0.0;
        for (int j = 0; j < dim; ++j) {
          const double g = (double)(float)sacc[j];
          sq += g * g;
        }
        s_sq = sq;
      }
      __syncthreads();
      const float Gn = __fadd_rn(row[wfl], (float)(s_sq / (double)dim));
      den = __fadd_rn(__fsqrt_rn(Gn), oa.eps);
      __syncthreads();
      if (threadIdx.x == 0) row[wfl] = Gn;
    }
    if (dim <= T) {
      if (pre) {
        const int j = threadIdx.x;
        const float g = (float)sacc[j];
        if (oa.opt == 0) {
          pw = sgd_w(pw, g, oa.lr);
        } else if (oa.opt == 1) {
          adagrad_step(pw, ps0, g, oa.lr, oa.eps);
          row[wfl + j] = ps0;
        } else if (oa.opt == 2) {
          adam_step(pw, ps0, ps1, g, oa);
          row[wfl + j] = ps0;
          row[wfl + dim + j] = ps1;
        } else {
          pw = __fsub_rn(pw, __fdiv_rn(__fmul_rn(oa.lr, g), den));
        }
        store_w(row, j, pw, bf16);
      }
    } else {
      for (int j = threadIdx.x; j < dim; j += T) update_col(row, dim, wfl, j, (float)sacc[j], oa, den);
    }
    __syncthreads();
  }
}

#endif  // DHS_TEMPLATES_ONLY

}  // namespace dhs
