// Forward kernels: lookup-or-insert, gather, in-order sum pooling, and the
// deterministic offset assignment of new keys.
//
// Pooling semantics: nn.EmbeddingBag(mode="sum") (DLRM practice article,
// section 2.1) over row lookups (RecIS background article, nn.Embedding
// section): pooled[b] = sum of the bag's rows, added in bag order in fp32.
//
// New keys are numbered by their first position in the batch.  The probe
// leaves PENDING | min position in the claimed slot; a bitmap over batch
// positions then marks each new key's first position, a prefix count over
// that bitmap gives its rank, and rank + row count is its row.  No kernel
// waits on another thread, and the map from keys to rows depends only on the
// key stream.
#pragma once

#include <climits>

#include "dhs_device.cuh"

// Bags of at least DHS_POOL_SPLIT_LEN ids on average are pooled by the split
// forward (a probe kernel with a thread per id, then fwd_pool_refs_kernel);
// shorter bags by the fused fwd_probe_pool_kernel.
#ifndef DHS_POOL_SPLIT_LEN
#define DHS_POOL_SPLIT_LEN 4
#endif
// Blocks per SM the fused pool kernel is compiled for with 32-lane groups
// and one 16-byte unit per lane (rows of 128 fp32 or 256 bf16 weights;
// register budget 65536 / (256 * blocks)); 4 at the other widths
#ifndef DHS_POOL_MINB
#define DHS_POOL_MINB 4
#endif

namespace dhs {

constexpr int kFwdThreads = 256;

// Bag ends of one chunk of G bags, held one per lane of the group and made
// safe to use: clamped into [start, n_keys] and non-decreasing.  Malformed
// offsets latch kErrInvalid.
template <int G>
__device__ __forceinline__ long long load_bag_ends(const long long* __restrict__ bag_off,
                                                   long long b0, int nb, long long n_keys,
                                                   long long n_bags, long long& start,
                                                   unsigned gmask, int gl, DevState* st) {
  long long s = __ldg(bag_off + b0);
  bool bad = false;
  if (b0 == 0 && s != 0) bad = true;
  if (s < 0 || s > n_keys) {
    bad = true;
    s = s < 0 ? 0 : n_keys;
  }
  long long e = (gl < nb) ? __ldg(bag_off + b0 + gl + 1) : n_keys;
  if (gl < nb) {
    if (e < s || e > n_keys) bad = true;
    if (b0 + gl + 1 == n_bags && e != n_keys) bad = true;
  }
  e = e < s ? s : (e > n_keys ? n_keys : e);
  // running max so that ends never decrease along the chunk
#pragma unroll
  for (int o = 1; o < G; o <<= 1) {
    const long long x = __shfl_up_sync(gmask, e, o, G);
    if (gl >= o && x > e) {
      e = x;
      bad = true;
    }
  }
  if (gl >= nb) e = LLONG_MAX;
  if (bad) latch(st, kErrInvalid);
  start = s;
  return e;
}

// A finished bag's accumulator as written out: mean pooling divides it by
// the bag's length (one rounded division; an empty bag stays 0).
template <bool MEAN>
__device__ __forceinline__ float4 bag_out(const float4& a, int len) {
  if (!MEAN || len <= 0) return a;
  const float fl = (float)len;
  return make_float4(__fdiv_rn(a.x, fl), __fdiv_rn(a.y, fl), __fdiv_rn(a.z, fl), __fdiv_rn(a.w, fl));
}

// Row units: a lane loads a row 16 bytes at a time; a unit holds 4 fp32
// weights, or 8 bf16 weights (BF) widened into two float4.
template <bool BF>
struct RowUnit {
  static constexpr int CV = BF ? 2 : 1;  // float4 per unit
  // unit c of the row at address r
  __device__ __forceinline__ static void load(unsigned long long r, int c, float4 (&x)[CV]) {
    if constexpr (BF) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(r) + c);
      unpack_bf16x8(u, x[0], x[CV - 1]);
    } else {
      x[0] = __ldg(reinterpret_cast<const float4*>(r) + c);
    }
  }
  // unit c of the initial row of `key`, as the assignment kernel stores it
  __device__ __forceinline__ static void init(unsigned long long key, int c, float4 (&x)[CV]) {
    if constexpr (BF) {
#pragma unroll
      for (int h = 0; h < CV; ++h) {
        const float4 v = init_weight4(key, c * 8 + 4 * h);
        x[h] = make_float4(round_bf16(v.x), round_bf16(v.y), round_bf16(v.z), round_bf16(v.w));
      }
    } else {
      x[0] = init_weight4(key, c * 4);
    }
  }
};

// Gather + pool of one window of cnt ids (kind, ref and weight held by lane t
// of the group for id t of the window): each lane loads NV units of U rows at
// a time, then adds them into the current bag's accumulator in id order,
// writing out each bag as its end is passed.  With NEW_KEYS, a new key's row
// is computed from the key, exactly as the assignment kernel stores it.  With
// W, each row is first multiplied by its id's weight (per-sample weights; one
// rounded product per element).  du: units per row (dim / 4, or dim / 8 for
// bf16 rows).
template <int G, int NV, bool NEW_KEYS, bool W, bool MEAN, bool BF>
__device__ __forceinline__ void pool_window(int kind, unsigned long long ref, float wt, int cnt, int ws,
                                            unsigned gmask, int gl, int du, int dim, int e,
                                            float4 (&acc)[NV * RowUnit<BF>::CV], int& cur, int& cur_end,
                                            int& cur_start, float* outb) {
  constexpr int CV = RowUnit<BF>::CV;
  constexpr int U = G < 8 / CV ? G : 8 / CV;
  for (int t0 = 0; t0 < cnt; t0 += U) {
    float4 v[U][NV * CV];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int t = t0 + u;
      const int src = t & (G - 1);
      const int kt = __shfl_sync(gmask, kind, src, G);
      const unsigned long long rt = __shfl_sync(gmask, ref, src, G);
      const float wtt = W ? __shfl_sync(gmask, wt, src, G) : 1.f;
#pragma unroll
      for (int q = 0; q < NV; ++q) {
        const int c = gl + q * G;
        float4 x[CV];
#pragma unroll
        for (int h = 0; h < CV; ++h) x[h] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (t < cnt && c < du) {
          if (kt == kHit)
            RowUnit<BF>::load(rt, c, x);
          else if (NEW_KEYS && kt == kNew)
            RowUnit<BF>::init(rt, c, x);
          if (W) {
#pragma unroll
            for (int h = 0; h < CV; ++h)
              x[h] = make_float4(__fmul_rn(wtt, x[h].x), __fmul_rn(wtt, x[h].y), __fmul_rn(wtt, x[h].z),
                                 __fmul_rn(wtt, x[h].w));
          }
        }
#pragma unroll
        for (int h = 0; h < CV; ++h) v[u][q * CV + h] = x[h];
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int t = t0 + u;
      if (t < cnt) {
        const int pos = ws + t;
        while (pos >= cur_end) {
          float4* o = reinterpret_cast<float4*>(outb + (long long)cur * dim);
#pragma unroll
          for (int q = 0; q < NV; ++q) {
            const int c = gl + q * G;
#pragma unroll
            for (int h = 0; h < CV; ++h) {
              // streamed: not read again here
              if (c < du) __stcs(o + c * CV + h, bag_out<MEAN>(acc[q * CV + h], cur_end - cur_start));
              acc[q * CV + h] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
          }
          ++cur;
          cur_start = cur_end;
          cur_end = __shfl_sync(gmask, e, cur & (G - 1), G);
        }
#pragma unroll
        for (int k = 0; k < NV * CV; ++k) acc[k] = f4add(acc[k], v[u][k]);
      }
    }
  }
}

// The bag in progress and the (empty) bags after it, at the end of a chunk.
template <int G, int NV, bool MEAN, bool BF>
__device__ __forceinline__ void flush_bags(float4 (&acc)[NV * RowUnit<BF>::CV], int cur, int nb, int cur_end,
                                           int cur_start, int gl, int du, int dim, float* outb) {
  constexpr int CV = RowUnit<BF>::CV;
  for (; cur < nb; ++cur) {
    float4* o = reinterpret_cast<float4*>(outb + (long long)cur * dim);
#pragma unroll
    for (int q = 0; q < NV; ++q) {
      const int c = gl + q * G;
#pragma unroll
      for (int h = 0; h < CV; ++h) {
        if (c < du) __stcs(o + c * CV + h, bag_out<MEAN>(acc[q * CV + h], cur_end - cur_start));
        acc[q * CV + h] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    cur_start = cur_end;  // later bags are empty: nothing to divide
  }
}

//   DHS_POOL_DYNAMIC  1: the fused pool kernel's groups take chunks of bags
//                     from a counter; 0: every ngroups-th chunk
#ifndef DHS_POOL_DYNAMIC
#define DHS_POOL_DYNAMIC 1
#endif

// The next chunk for a group of G lanes, from the call's counter.
__device__ __forceinline__ int pool_fetch(unsigned* ctr, unsigned gmask, int gl, int G) {
  unsigned c = 0;
  if (gl == 0) c = atomicAdd(ctr, 1u);
  return (int)__shfl_sync(gmask, c, 0, G);
}

// Fused lookup-or-insert + gather + sum pooling.  A group of G lanes owns a
// chunk of G consecutive bags; it probes the chunk's ids G at a time (one id
// per lane; the probing lane also forms the row address), then walks those ids
// in order, each lane loading NV float4 columns of the row (16-byte vector
// loads), U rows in flight, and adds them into the current bag's accumulator.
// A new key's row is not read: its initial value is computed from the key,
// exactly as the assignment kernel will store it.  Pooling form PM: 0 sum,
// 1 sum with per-sample weights psw[position] scaling each row, 2 mean
// (each bag divided by its length).  BF: the table's weights are bf16.
template <int G, int NV, int PM, bool BF>
__global__ void __launch_bounds__(kFwdThreads, NV == 1 ? (G == 32 ? DHS_POOL_MINB : 4) : (NV == 2 ? 2 : 1))
fwd_probe_pool_kernel(IdMap m, RowSpace rs, int dim, const long long* __restrict__ keys,
                      long long n_keys, const long long* __restrict__ bag_off, long long n_bags,
                      const float* __restrict__ psw,
                      float* __restrict__ out, unsigned* __restrict__ nbm,
                      unsigned* __restrict__ slotpos, int ctr_sel, DevState* st) {
  pdl_enter();
  constexpr bool W = PM == 1, MEAN = PM == 2;
  const int lane = threadIdx.x & 31;
  const int gl = lane & (G - 1);
  const int gw = lane / G;
  const unsigned gmask = (G == 32) ? 0xffffffffu : (((1u << G) - 1u) << (gw * G));
  const int gid = (int)((blockIdx.x * kFwdThreads + threadIdx.x) / G);
  const int ngroups = (int)((gridDim.x * kFwdThreads) / G);
  // bags and positions fit in 31 bits (the host rejects larger calls)
  const int nchunks = (int)((n_bags + G - 1) / G);
  constexpr int CV = RowUnit<BF>::CV;
  const int du = BF ? dim >> 3 : dim >> 2;  // 16-byte units of a row's weights

#if DHS_POOL_DYNAMIC
  // chunks handed out one at a time from this call's counter, so that groups
  // whose chunks take longer take fewer; the next call's counter is cleared
  unsigned* const ctr = &st->fwd_ctr[ctr_sel];
  if (blockIdx.x == 0 && threadIdx.x == 0) st->fwd_ctr[ctr_sel ^ 1] = 0u;
  for (int c = pool_fetch(ctr, gmask, gl, G); c < nchunks; c = pool_fetch(ctr, gmask, gl, G)) {
#else
  for (int c = gid; c < nchunks; c += ngroups) {
#endif
    const long long b0 = (long long)c * G;
    const int nb = (int)min((long long)G, n_bags - b0);
    long long s64;
    const long long e64 = load_bag_ends<G>(bag_off, b0, nb, n_keys, n_bags, s64, gmask, gl, st);
    const int e = e64 == LLONG_MAX ? INT_MAX : (int)e64;
    const int s = (int)s64;
    const int E = __shfl_sync(gmask, e, nb - 1, G);
    int cur = 0, cur_start = s;
    int cur_end = __shfl_sync(gmask, e, 0, G);
    float4 acc[NV * CV];
#pragma unroll
    for (int q = 0; q < NV * CV; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    float* outb = out + b0 * (long long)dim;

    for (int ws = s; ws < E; ws += G) {
      const int cnt = min(G, E - ws);
      // ---- probe: one id per lane ----
      // ref: the row address of a hit, or the key itself for a new key
      int kind = kBad;
      unsigned long long ref = 0;
      float wt = 0.f;
      if (gl < cnt) {
        const int p = ws + gl;
        const long long k = __ldg(keys + p);
        if (W) wt = __ldg(psw + p);
        if (k < 0) {
          latch(st, kErrInvalid);
        } else {
          unsigned long long r;
          kind = probe_claim(m, (unsigned long long)k, (unsigned)p, r, st);
          if (kind == kHit) {
            const float* rowp = rs.row(r);
            ref = (unsigned long long)rowp;
            prefetch_l2(rowp, (unsigned)dim * (BF ? 2u : 4u));  // all G rows of the window in flight
          } else if (kind == kNew) {
            slotpos[p] = (unsigned)r;
            ref = (unsigned long long)k;
          }
        }
      }
      // mark the positions that carry a key new in this call (<= 2 words per window)
      {
        const unsigned bal = __ballot_sync(gmask, kind == kNew);
        const unsigned mine = (G == 32) ? bal : ((bal >> (gw * G)) & ((1u << G) - 1u));
        if (gl == 0 && mine) {
          const unsigned p0 = (unsigned)ws;
          const unsigned sh = p0 & 31u;
          atomicOr(&nbm[p0 >> 5], mine << sh);
          if (sh && (sh + G > 32)) {
            const unsigned hi = mine >> (32 - sh);
            if (hi) atomicOr(&nbm[(p0 >> 5) + 1], hi);
          }
        }
      }
      pool_window<G, NV, true, W, MEAN, BF>(kind, ref, wt, cnt, ws, gmask, gl, du, dim, e, acc, cur, cur_end,
                                            cur_start, outb);
    }
    // the bag in progress and any empty bags after it
    flush_bags<G, NV, MEAN, BF>(acc, cur, nb, cur_end, cur_start, gl, du, dim, outb);
  }
}

// Gather + pool from per-id row references (the split forward for long bags,
// run after the new keys' rows are assigned and written): refs[p] >= 0 is the
// row of a hit, <= -2 the slot -(2 + refs[p]) of a key new in this call (its
// row is the slot's value), -1 an id without a row.  The references of the
// window two ahead (and the slot values of the next window's new ids) are
// loaded while the current window is gathered, so no window waits on a probe.
// Bags, windows and the order of additions are those of fwd_probe_pool_kernel,
// and so is the pooling form PM.  The reference of a new key's position is
// replaced by its row (kRecNoRow: none), so that after the call refs[p] is
// the row of position p for every key that has one.
template <int G, int NV, int PM, bool BF>
__global__ void __launch_bounds__(kFwdThreads, NV == 1 ? 4 : (NV == 2 ? 2 : 1))
fwd_pool_refs_kernel(RowSpace rs, int dim, const Slot* __restrict__ slots,
                     long long* __restrict__ refs, long long n_keys,
                     const long long* __restrict__ bag_off, long long n_bags,
                     const float* __restrict__ psw,
                     float* __restrict__ out, DevState* st) {
  pdl_enter();
  constexpr bool W = PM == 1, MEAN = PM == 2;
  const int lane = threadIdx.x & 31;
  const int gl = lane & (G - 1);
  const int gw = lane / G;
  const unsigned gmask = (G == 32) ? 0xffffffffu : (((1u << G) - 1u) << (gw * G));
  const int gid = (int)((blockIdx.x * kFwdThreads + threadIdx.x) / G);
  const int ngroups = (int)((gridDim.x * kFwdThreads) / G);
  const int nchunks = (int)((n_bags + G - 1) / G);
  constexpr int CV = RowUnit<BF>::CV;
  const int du = BF ? dim >> 3 : dim >> 2;  // 16-byte units of a row's weights

  for (int c = gid; c < nchunks; c += ngroups) {
    const long long b0 = (long long)c * G;
    const int nb = (int)min((long long)G, n_bags - b0);
    long long s64;
    const long long e64 = load_bag_ends<G>(bag_off, b0, nb, n_keys, n_bags, s64, gmask, gl, st);
    const int e = e64 == LLONG_MAX ? INT_MAX : (int)e64;
    const int s = (int)s64;
    const int E = __shfl_sync(gmask, e, nb - 1, G);
    int cur = 0, cur_start = s;
    int cur_end = __shfl_sync(gmask, e, 0, G);
    float4 acc[NV * CV];
#pragma unroll
    for (int q = 0; q < NV * CV; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    float* outb = out + b0 * (long long)dim;

    auto ref_at = [&](int p) -> long long { return p < E ? refs[p] : -1; };
    auto w_at = [&](int p) -> float { return (W && p < E) ? __ldg(psw + p) : 0.f; };
    long long r0 = ref_at(s + gl), r1 = ref_at(s + G + gl);
    float w0 = w_at(s + gl);
    // the row of a new key (PENDING if its assignment failed: the table is full)
    auto new_row = [&](long long r) -> unsigned long long {
      return r <= -2 ? __ldg(&slots[-2 - r].val) : kPending;
    };
    unsigned long long n0 = new_row(r0);
    for (int ws = s; ws < E; ws += G) {
      const int cnt = min(G, E - ws);
      const long long rc = r0;
      const unsigned long long nc = n0;
      const float wc = w0;
      r0 = r1;
      r1 = ref_at(ws + 2 * G + gl);
      n0 = new_row(r0);
      if (W) w0 = w_at(ws + G + gl);
      int kind = kBad;
      unsigned long long ref = 0;
      if (gl < cnt) {
        if (rc >= 0) {
          kind = kHit;
          ref = (unsigned long long)rs.row((unsigned long long)rc);
        } else if (rc <= -2) {
          if (!(nc & kPending)) {
            kind = kHit;
            ref = (unsigned long long)rs.row(nc);
          }
          // the reference left for the backward: the row, or no row
          refs[ws + gl] = (nc & kPending) ? kRecNoRow : (long long)nc;
        }
      }
      pool_window<G, NV, false, W, MEAN, BF>(kind, ref, wc, cnt, ws, gmask, gl, du, dim, e, acc, cur, cur_end,
                                             cur_start, outb);
    }
    flush_bags<G, NV, MEAN, BF>(acc, cur, nb, cur_end, cur_start, gl, du, dim, outb);
  }
}

#ifndef DHS_TEMPLATES_ONLY
// Lookup-or-insert without pooling: thread per position.  offsets_out holds
// the row offset of a hit, -(2 + slot) for a key without a row yet (new in
// this call, or not admitted: resolved by fwd_fixup_kernel or by the gather)
// and -1 for a negative key.  With hooks, every key's slot is stamped with
// the call's step, a key without a row has its occurrence counted, and the
// slots taken from empty are counted in keys_used.  rec_keys (may be null)
// gets a copy of the keys: with offsets_out (once fwd_pool_refs_kernel has
// put the new keys' rows in) it is the call's record of key and row per
// position, which a backward on the same keys reads instead of probing.
__global__ void __launch_bounds__(kFwdThreads)
fwd_probe_offsets_kernel(IdMap m, const long long* __restrict__ keys, long long n,
                         long long* __restrict__ offsets_out, unsigned* __restrict__ nbm,
                         unsigned* __restrict__ slotpos, long long* __restrict__ rec_keys, Hooks hk,
                         DevState* st) {
  pdl_enter();
  const long long p = (long long)blockIdx.x * kFwdThreads + threadIdx.x;
  bool is_new = false, claimed = false;
  if (p < n) {
    const long long k = __ldg(keys + p);
    if (rec_keys) rec_keys[p] = k;
    long long o = -1;
    if (k < 0) {
      latch(st, kErrInvalid);
    } else {
      unsigned long long ref, slot;
      const int kind = probe_claim(m, (unsigned long long)k, (unsigned)p, ref, slot, claimed, st);
      if (kind == kHit) {
        o = (long long)ref;
      } else if (kind == kNew) {
        o = -2 - (long long)ref;
        slotpos[p] = (unsigned)ref;
        is_new = true;
        if (hk.cnt) atomicAdd(hk.cnt + slot, 1u);
      }
      if (hk.stamp && kind != kBad && hk.stamp[slot] != hk.step) hk.stamp[slot] = hk.step;
    }
    offsets_out[p] = o;
  }
  // positions of a warp are one aligned 32-bit word of the bitmap
  const unsigned bal = __ballot_sync(0xffffffffu, is_new);
  if ((threadIdx.x & 31) == 0 && bal) nbm[p >> 5] = bal;
  if (hk.cnt || hk.stamp) {
    const unsigned cb = __ballot_sync(0xffffffffu, claimed);
    if ((threadIdx.x & 31) == 0 && cb) atomicAdd(&st->keys_used, (unsigned long long)__popc(cb));
  }
}

__global__ void fwd_fixup_kernel(const Slot* __restrict__ slots, long long* __restrict__ offsets,
                                 long long n) {
  pdl_enter();
  for (long long p = (long long)blockIdx.x * blockDim.x + threadIdx.x; p < n;
       p += (long long)gridDim.x * blockDim.x) {
    const long long o = offsets[p];
    if (o <= -2) {
      const unsigned long long v = slots[-2 - o].val;
      offsets[p] = (v & kPending) ? -1 : (long long)v;  // no row: not admitted
    }
  }
}

// First-occurrence marking.  Block of 1024 threads per group of 4096 batch
// positions (128 bitmap words), four positions per thread so that each thread
// has four independent load chains in flight.  A position that carries a key
// new in this call is its key's first occurrence iff the key's slot holds
// PENDING | that position.  Writes the first-occurrence bitmap words, clears
// the new-position words for the next call, and writes the group's count.
// With admission, a first occurrence whose key has been seen fewer times than
// the threshold gets no row (its slot goes back to COUNTING).  The last block
// to finish scans the group counts, reserves the new rows (the first ones
// from the free list, the rest appended: row_base = row_count, row_count +=
// M - taken) and resets the ticket.
constexpr int kGroupThreads = 1024;
constexpr int kGroupPerThread = 4;
constexpr int kGroupPositions = kGroupThreads * kGroupPerThread;  // 4096
constexpr int kGroupWords = kGroupPositions / 32;                  // 128

__global__ void __launch_bounds__(kGroupThreads)
fwd_mark_kernel(Slot* __restrict__ slots, unsigned* __restrict__ nbm,
                unsigned* __restrict__ fbm, unsigned* __restrict__ gcnt,
                unsigned* __restrict__ gpref, const unsigned* __restrict__ slotpos,
                long long nwords, long long ngroups, Hooks hk, DevState* st) {
  pdl_enter();
  __shared__ unsigned wsum[32];
  __shared__ bool is_last;
  __shared__ unsigned long long carry_s;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const long long g = blockIdx.x;
  unsigned word[kGroupPerThread];
  unsigned s[kGroupPerThread];
  unsigned long long v[kGroupPerThread];
#pragma unroll
  for (int k = 0; k < kGroupPerThread; ++k) {
    const long long w = g * kGroupWords + k * 32 + wid;
    word[k] = w < nwords ? nbm[w] : 0u;
  }
#pragma unroll
  for (int k = 0; k < kGroupPerThread; ++k) {
    const unsigned long long p = (unsigned long long)(g * kGroupPositions + k * kGroupThreads + threadIdx.x);
    s[k] = ((word[k] >> lane) & 1u) ? slotpos[p] : 0u;
  }
#pragma unroll
  for (int k = 0; k < kGroupPerThread; ++k)
    v[k] = ((word[k] >> lane) & 1u) ? __ldcg(&slots[s[k]].val) : 0ull;
  unsigned cnt = 0;
#pragma unroll
  for (int k = 0; k < kGroupPerThread; ++k) {
    const long long w = g * kGroupWords + k * 32 + wid;
    const unsigned long long p = (unsigned long long)(g * kGroupPositions + k * kGroupThreads + threadIdx.x);
    bool first = ((word[k] >> lane) & 1u) && (v[k] & ~kPending) == p;
    if (first && hk.admit > 1 && hk.cnt[s[k]] < hk.admit) {
      slots[s[k]].val = kCounting;  // seen too few times: no row yet
      first = false;
    }
    const unsigned fw = __ballot_sync(0xffffffffu, first);
    if (lane == 0 && w < nwords) {
      fbm[w] = fw;
      if (word[k]) nbm[w] = 0u;
    }
    cnt += __popc(fw);
  }
  if (lane == 0) wsum[wid] = cnt;
  __syncthreads();
  if (wid == 0) {
    const unsigned c = warp_sum_u32(wsum[lane]);
    if (lane == 0) gcnt[g] = c;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(&st->ticket, 1u) == gridDim.x - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();

  // exclusive scan of gcnt[0, ngroups) by this block, 1024 entries per pass
  if (threadIdx.x == 0) carry_s = 0;
  __syncthreads();
  for (long long base = 0; base < ngroups; base += kGroupThreads) {
    const long long i = base + threadIdx.x;
    const unsigned x = (i < ngroups) ? __ldcg(gcnt + i) : 0u;
    unsigned inc = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    if (lane == 31) wsum[wid] = inc;
    __syncthreads();
    if (wid == 0) {
      const unsigned vv = wsum[lane];
      unsigned vi = vv;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, vi, o);
        if (lane >= o) vi += y;
      }
      wsum[lane] = vi - vv;  // exclusive prefix of the warp sums
    }
    __syncthreads();
    const unsigned long long carry = carry_s;
    if (i < ngroups) gpref[i] = (unsigned)(carry + wsum[wid] + inc - x);
    __syncthreads();
    if (threadIdx.x == kGroupThreads - 1) carry_s = carry + wsum[wid] + inc;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    // new rows come from the free list (evicted rows, ascending) first, then
    // are appended
    const unsigned long long M = carry_s;
    const unsigned long long avail = st->free_count - st->free_head;
    const unsigned long long use = M < avail ? M : avail;
    st->free_base = st->free_head;
    st->m_free = use;
    st->free_head += use;
    const unsigned long long base = st->row_count;
    st->row_base = base;
    st->row_count = base + (M - use);
    st->m_last = M;
    st->sum_new += M;
    st->ticket = 0u;
    __threadfence();
  }
}

// Offset assignment + row initialisation of group g (4096 batch positions,
// 1024 threads): the group's new keys have consecutive ranks from rank0 (the
// prefix over the group's 128 first-occurrence words, fw_of(word), plus the
// bit's place in its word), so their rows are one contiguous run.  Each
// first occurrence's row offset goes into its slot; the run is written with
// coalesced 16-byte stores (initial weights from splitmix64(key), optimizer
// state zero).  Rank q takes free-list row free_list[free_base + q] while
// q < m_free, else appended row row_base + (q - m_free).
#ifndef DHS_ASSIGN_COLUMNS
#define DHS_ASSIGN_COLUMNS 1  // column-per-thread row initialisation (0: flat index loop only)
#endif

template <class FW>
__device__ __forceinline__ void assign_group(long long g, FW fw_of, unsigned long long rank0,
                                             unsigned long long m_free, unsigned long long free_base,
                                             unsigned long long row_base, Slot* __restrict__ slots,
                                             RowSpace rs, int dim, const long long* __restrict__ keys,
                                             const unsigned* __restrict__ slotpos, long long nwords, Hooks hk,
                                             DevState* st, unsigned long long* skey, unsigned* wpre,
                                             unsigned* s_total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (threadIdx.x < 32) {
    // exclusive prefix of the 128 words' counts (4 per lane, in word order)
    unsigned c[4], t = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const long long w = g * kGroupWords + lane * 4 + k;
      c[k] = w < nwords ? __popc(fw_of(w)) : 0u;
      t += c[k];
    }
    unsigned inc = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    unsigned run = inc - t;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      wpre[lane * 4 + k] = run;
      run += c[k];
    }
    if (lane == 31) *s_total = inc;
  }
  __syncthreads();
  const unsigned total = *s_total;
  const unsigned r_lo = 0, r_hi = total;  // the group's rows
  // rank q of the call's new keys: free-list row q while q < m_free, else
  // appended row row_base + (q - m_free)
  auto row_of = [&](unsigned long long q) -> unsigned long long {
    return q < m_free ? (unsigned long long)hk.free_list[free_base + q] : row_base + (q - m_free);
  };
  const unsigned long long limit = st->n_blocks << rs.log2_br;
#pragma unroll
  for (int k = 0; k < kGroupPerThread; ++k) {
    const int wi = k * 32 + wid;
    const long long w = g * kGroupWords + wi;
    const unsigned fw = w < nwords ? fw_of(w) : 0u;
    if ((fw >> lane) & 1u) {
      const unsigned j = wpre[wi] + __popc(fw & lanemask_lt());
      const unsigned long long p = (unsigned long long)(g * kGroupPositions + k * kGroupThreads + threadIdx.x);
      if (j >= r_lo && j < r_hi) skey[j] = (unsigned long long)__ldg(keys + p);  // the key first seen at p
      {
        const unsigned sl = slotpos[p];
        const unsigned long long row = row_of(rank0 + j);
        if (rank0 + j < m_free) atomicAnd(hk.free_bm + (row >> 5), ~(1u << (row & 31)));  // no longer free
        if (row < limit) {
          slots[sl].val = row;
        } else {
          latch(st, kErrFull);
          slots[sl].val = kPending;  // unusable; the table is reported full
        }
      }
    }
  }
  __syncthreads();
  const int s4 = rs.stride >> 2;
  const int du = rs.wfl >> 2;  // 16-byte units holding the weights (4 fp32 or 8 bf16 each)
  const bool bf = rs.wfl != dim;
  const int work = (int)(r_hi - r_lo) * s4;
  // idx / s4 as a multiply-high by ceil(2^32 / s4) (s4 >= 2; that does not fit
  // 32 bits for s4 = 1): exact while idx * s4 < 2^32 (here idx < 4096 * s4 and
  // s4 <= 384)
  const unsigned inv = s4 > 1 ? (unsigned)((0x100000000ull + (unsigned)s4 - 1) / (unsigned)s4) : 0u;
  // appended rows are one contiguous run: rows before the first block edge
  // share one base pointer; free-list rows are placed one by one
  const unsigned long long qfirst = rank0 + r_lo;
  const bool contiguous = qfirst >= m_free;
  const unsigned long long rfirst = contiguous ? row_of(qfirst) : 0;
#if DHS_ASSIGN_COLUMNS
  // Common case: appended rows, all below the limit, and a row's 16-byte
  // units (weights, then state) dividing the block's threads.  Each thread
  // then keeps one column of the run (its hash offset loop-invariant) and
  // steps over rows, one EmbeddingBlock piece of the run at a time.
  const int nrows = (int)(r_hi - r_lo), sd = s4 - du;
  if (contiguous && rfirst + (unsigned long long)nrows <= limit && du <= kGroupThreads &&
      kGroupThreads % du == 0 && (sd == 0 || (sd <= kGroupThreads && kGroupThreads % sd == 0))) {
    const int wc = threadIdx.x % du, wstep = kGroupThreads / du;
    for (int r0 = 0; r0 < nrows;) {
      const unsigned long long row0 = rfirst + (unsigned long long)r0;
      const int len = (int)min((unsigned long long)(nrows - r0), (rs.br_mask + 1) - (row0 & rs.br_mask));
      float4* const b = reinterpret_cast<float4*>(rs.row(row0));
      const unsigned long long* const kr = skey + r_lo + r0;
      if (!bf) {
        for (int r = threadIdx.x / du; r < len; r += wstep) b[(size_t)r * s4 + wc] = init_weight4(kr[r], wc * 4);
      } else {
        for (int r = threadIdx.x / du; r < len; r += wstep) {
          const float4 a = init_weight4(kr[r], wc * 8), c = init_weight4(kr[r], wc * 8 + 4);
          reinterpret_cast<uint4*>(b)[(size_t)r * s4 + wc] =
              make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(c.x, c.y), pack_bf16x2(c.z, c.w));
        }
      }
      if (sd > 0) {
        const int sc = threadIdx.x % sd, sstep = kGroupThreads / sd;
        for (int r = threadIdx.x / sd; r < len; r += sstep) b[(size_t)r * s4 + du + sc] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      r0 += len;
    }
    return;
  }
#endif
  const unsigned long long in_block = (rs.br_mask + 1) - (rfirst & rs.br_mask);
  float4* const base = contiguous && rfirst < limit ? reinterpret_cast<float4*>(rs.row(rfirst)) : nullptr;
  for (int idx = threadIdx.x; idx < work; idx += kGroupThreads) {
    const int r = s4 > 1 ? (int)__umulhi((unsigned)idx, inv) : idx;
    const int c4 = idx - r * s4;
    const unsigned long long row = contiguous ? rfirst + r : row_of(qfirst + r);
    if (row >= limit) continue;
    float4* dst = contiguous && (unsigned long long)r < in_block ? base + (size_t)r * s4
                                                                 : reinterpret_cast<float4*>(rs.row(row));
    if (c4 >= du) {
      dst[c4] = make_float4(0.f, 0.f, 0.f, 0.f);
    } else if (!bf) {
      dst[c4] = init_weight4(skey[r_lo + r], c4 * 4);
    } else {
      const float4 a = init_weight4(skey[r_lo + r], c4 * 8), b = init_weight4(skey[r_lo + r], c4 * 8 + 4);
      reinterpret_cast<uint4*>(dst)[c4] =
          make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
    }
  }
}

// The two-kernel form (first-occurrence marking by fwd_mark_kernel, whose
// last block scans the group counts and reserves the rows): one block per
// group.  More blocks per group (each writing a share of the run) measured
// slower: each repeated the prefix and the key gathering for fewer rows.
__global__ void __launch_bounds__(kGroupThreads, 2)
fwd_assign_kernel(Slot* __restrict__ slots, RowSpace rs, int dim, const long long* __restrict__ keys,
                  const unsigned* __restrict__ fbm, const unsigned* __restrict__ gpref,
                  const unsigned* __restrict__ slotpos, long long nwords, long long ngroups,
                  Hooks hk, DevState* st) {
  pdl_enter();
  __shared__ unsigned long long skey[kGroupPositions];  // 32 KB
  __shared__ unsigned wpre[kGroupWords];
  __shared__ unsigned s_total;
  const long long g = blockIdx.x;
  auto fw_of = [&](long long w) -> unsigned { return fbm[w]; };
  assign_group(g, fw_of, (unsigned long long)gpref[g], st->m_free, st->free_base, st->row_base, slots, rs, dim,
               keys, slotpos, nwords, hk, st, skey, wpre, &s_total);
}

// ---- IDMap maintenance and read-only access ----

__global__ void fill_empty_kernel(Slot* __restrict__ slots, unsigned long long n) {
  for (unsigned long long i = (unsigned long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (unsigned long long)gridDim.x * blockDim.x)
    reinterpret_cast<ulonglong2*>(slots)[i] = make_ulonglong2(kEmptyKey, kEmptyKey);
}

// Re-insert every key of `from` into the empty map `to` (keys are distinct,
// offsets keep their values: rows never move); tombstones are dropped.  With
// hooks the per-slot counts and stamps move with their keys, and the keys
// placed are counted in keys_used (zero on entry).
__global__ void rehash_kernel(const Slot* __restrict__ from, unsigned long long n_from, IdMap to,
                              const unsigned* __restrict__ from_cnt, unsigned* __restrict__ to_cnt,
                              const unsigned* __restrict__ from_stamp, unsigned* __restrict__ to_stamp,
                              DevState* st) {
  // every lane of a warp runs the same iterations (full-warp ballots below)
  const unsigned long long stride = (unsigned long long)gridDim.x * blockDim.x;
  for (unsigned long long i0 = (unsigned long long)blockIdx.x * blockDim.x; i0 < n_from; i0 += stride) {
    const unsigned long long i = i0 + threadIdx.x;
    const ulonglong2 sv = i < n_from ? reinterpret_cast<const ulonglong2*>(from)[i]
                                     : make_ulonglong2(kEmptyKey, kEmptyKey);
    bool placed = false;
    if (sv.x != kEmptyKey && sv.x != kTombKey) {
      unsigned long long w = hash_key(sv.x) & to.win_mask;
      for (unsigned long long step = 0; step <= to.win_mask && !placed; ++step) {
        Slot* ws = to.slots + 2 * w;
        for (int j = 0; j < 2 && !placed; ++j) {
          if (atomicCAS(&ws[j].key, kEmptyKey, sv.x) == kEmptyKey) {
            ws[j].val = sv.y;
            const unsigned long long at = 2 * w + j;
            if (to_cnt) to_cnt[at] = from_cnt[i];
            if (to_stamp) to_stamp[at] = from_stamp[i];
            placed = true;
          }
        }
        w = (w + 1) & to.win_mask;
      }
      if (!placed) latch(st, kErrFull);
    }
    if (to_cnt || to_stamp) {
      const unsigned b = __ballot_sync(0xffffffffu, placed);
      if ((threadIdx.x & 31) == 0 && b) atomicAdd(&st->keys_used, (unsigned long long)__popc(b));
    }
  }
}

// ---- eviction ----

// Every key last seen before step keep_from becomes a tombstone; the row of
// a key that had one is marked free.  freed counts the rows freed.
__global__ void evict_kernel(Slot* __restrict__ slots, unsigned long long n, const unsigned* __restrict__ stamp,
                             unsigned keep_from, unsigned* __restrict__ free_bm,
                             unsigned long long* __restrict__ freed) {
  const unsigned long long stride = (unsigned long long)gridDim.x * blockDim.x;
  for (unsigned long long i0 = (unsigned long long)blockIdx.x * blockDim.x; i0 < n; i0 += stride) {
    const unsigned long long i = i0 + threadIdx.x;
    const ulonglong2 sv = i < n ? reinterpret_cast<const ulonglong2*>(slots)[i] : make_ulonglong2(kEmptyKey, kEmptyKey);
    bool freed_row = false;
    if (sv.x != kEmptyKey && sv.x != kTombKey && stamp[i] < keep_from) {
      if (!(sv.y & kPending)) {
        atomicOr(free_bm + (sv.y >> 5), 1u << (sv.y & 31));
        freed_row = true;
      }
      reinterpret_cast<ulonglong2*>(slots)[i] = make_ulonglong2(kTombKey, kTombKey);
    }
    const unsigned b = __ballot_sync(0xffffffffu, freed_row);
    if ((threadIdx.x & 31) == 0 && b) atomicAdd(freed, (unsigned long long)__popc(b));
  }
}

// Free list from the free-row bitmap, ascending, in two launches.  Count: a
// block per kFreeWords words writes its count of free rows; the last block to
// finish turns the counts into exclusive offsets, sets free_count and resets
// free_head.  Scatter: each block writes its rows from its offset.
constexpr int kFreeThreads = 1024;
constexpr int kFreeWords = kFreeThreads;  // one bitmap word per thread

__global__ void __launch_bounds__(kFreeThreads)
free_count_kernel(const unsigned* __restrict__ free_bm, long long nwords, unsigned* __restrict__ bcnt,
                  long long nblocks, DevState* st) {
  __shared__ unsigned wsum[32];
  __shared__ bool is_last;
  __shared__ unsigned long long carry_s;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const long long w = (long long)blockIdx.x * kFreeWords + threadIdx.x;
  const unsigned c = warp_sum_u32(w < nwords ? __popc(free_bm[w]) : 0u);
  if (lane == 0) wsum[wid] = c;
  __syncthreads();
  if (wid == 0) {
    const unsigned t = warp_sum_u32(wsum[lane]);
    if (lane == 0) bcnt[blockIdx.x] = t;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = atomicAdd(&st->ticket2, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  if (threadIdx.x == 0) carry_s = 0;
  __syncthreads();
  for (long long b0 = 0; b0 < nblocks; b0 += kFreeThreads) {
    const long long i = b0 + threadIdx.x;
    const unsigned x = i < nblocks ? __ldcg(bcnt + i) : 0u;
    unsigned inc = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    if (lane == 31) wsum[wid] = inc;
    __syncthreads();
    if (wid == 0) {
      const unsigned vv = wsum[lane];
      unsigned vi = vv;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, vi, o);
        if (lane >= o) vi += y;
      }
      wsum[lane] = vi - vv;
    }
    __syncthreads();
    const unsigned long long carry = carry_s;
    if (i < nblocks) bcnt[i] = (unsigned)(carry + wsum[wid] + inc - x);
    __syncthreads();
    if (threadIdx.x == kFreeThreads - 1) carry_s = carry + wsum[wid] + inc;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    st->free_count = carry_s;
    st->free_head = 0;
    st->ticket2 = 0u;
    __threadfence();
  }
}

__global__ void __launch_bounds__(kFreeThreads)
free_scatter_kernel(const unsigned* __restrict__ free_bm, long long nwords, const unsigned* __restrict__ boff,
                    unsigned* __restrict__ free_list) {
  __shared__ unsigned wsum[32];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const long long w = (long long)blockIdx.x * kFreeWords + threadIdx.x;
  unsigned bits = w < nwords ? free_bm[w] : 0u;
  const unsigned c = __popc(bits);
  unsigned inc = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) wsum[wid] = inc;
  __syncthreads();
  if (wid == 0) {
    const unsigned vv = wsum[lane];
    unsigned vi = vv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned y = __shfl_up_sync(0xffffffffu, vi, o);
      if (lane >= o) vi += y;
    }
    wsum[lane] = vi - vv;
  }
  __syncthreads();
  unsigned at = boff[blockIdx.x] + wsum[wid] + inc - c;
  while (bits) {
    const int b = __ffs(bits) - 1;
    free_list[at++] = (unsigned)(w * 32 + b);
    bits &= bits - 1;
  }
}

__global__ void lookup_kernel(IdMap m, const long long* __restrict__ keys, long long n,
                              long long* __restrict__ out) {
  pdl_enter();
  for (long long p = (long long)blockIdx.x * blockDim.x + threadIdx.x; p < n;
       p += (long long)gridDim.x * blockDim.x) {
    const long long k = __ldg(keys + p);
    const long long o = k < 0 ? -1 : probe_find(m, (unsigned long long)k);
    out[p] = o < 0 ? -1 : o;
  }
}

// Full rows of the given keys as fp32 (weights widened from bf16 where the
// table stores bf16), ostride = dim + state floats per output row; warp per
// key, NaN for an absent key.
__global__ void get_rows_kernel(IdMap m, RowSpace rs, int dim, int ostride, const long long* __restrict__ keys,
                                long long n, float* __restrict__ out) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  const bool bf = rs.wfl != dim;
  const float nan = __int_as_float(0x7fc00000);
  for (long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < n; i += nw) {
    const long long k = __ldg(keys + i);
    const long long off = k < 0 ? -1 : probe_find(m, (unsigned long long)k);
    float* o = out + i * (long long)ostride;
    const float* row = off < 0 ? nullptr : rs.row((unsigned long long)off);
    for (int j = lane; j < ostride; j += 32) {
      float v = nan;
      if (row) {
        if (j >= dim)
          v = row[rs.wfl + (j - dim)];
        else
          v = bf ? __uint_as_float((unsigned)reinterpret_cast<const unsigned short*>(row)[j] << 16) : row[j];
      }
      o[j] = v;
    }
  }
}

// keys_by_row[val] = key for every occupied slot (export in row order).
__global__ void keys_by_row_kernel(const Slot* __restrict__ slots, unsigned long long n,
                                   long long* __restrict__ keys_by_row, unsigned long long rows) {
  for (unsigned long long i = (unsigned long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (unsigned long long)gridDim.x * blockDim.x) {
    const ulonglong2 sv = reinterpret_cast<const ulonglong2*>(slots)[i];
    if (sv.x != kEmptyKey && sv.y < rows) keys_by_row[sv.y] = (long long)sv.x;
  }
}

__global__ void pack_keys_kernel(const int* __restrict__ tids, const long long* __restrict__ ids,
                                 long long n, long long* __restrict__ keys) {
  pdl_enter();
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const long long t = tids[i], id = ids[i];
    const bool ok = t >= 0 && t < (1 << 15) && id >= 0 && id < (1ll << 48);
    keys[i] = ok ? ((t << 48) | id) : -1;
  }
}

#endif  // DHS_TEMPLATES_ONLY

}  // namespace dhs
