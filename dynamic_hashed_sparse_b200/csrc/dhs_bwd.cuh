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
// more sort chunks (a hot key) is summed in pieces by every chunk it covers
// and the pieces are combined by one thread block.
#pragma once

#include "dhs_device.cuh"

namespace dhs {

// ---------------------------------------------------------------------------
// probe: (row, bag) of every position, bag-major order
// ---------------------------------------------------------------------------

#ifndef DHS_TEMPLATES_ONLY
// Warp per chunk of 32 bags; positions 32 at a time, one per lane.  A lane
// finds its bag by counting the chunk's bag ends at or before its position.
// Missing or negative keys get row `sentinel` (sorted last, never updated).
__global__ void __launch_bounds__(256)
bwd_probe_kernel(IdMap m, const long long* __restrict__ keys, long long n_keys,
                 const long long* __restrict__ bag_off, long long n_bags,
                 unsigned* __restrict__ rkey, unsigned* __restrict__ rval, unsigned sentinel,
                 DevState* st) {
  const int lane = threadIdx.x & 31;
  const long long nchunks = (n_bags + 31) / 32;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long c = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; c < nchunks;
       c += nw) {
    const long long b0 = c * 32;
    const int nb = (int)min(32ll, n_bags - b0);
    long long s = __ldg(bag_off + b0);
    bool bad = (b0 == 0 && s != 0) || s < 0 || s > n_keys;
    s = s < 0 ? 0 : (s > n_keys ? n_keys : s);
    long long e = lane < nb ? __ldg(bag_off + b0 + lane + 1) : n_keys;
    if (lane < nb && (e < s || e > n_keys || (b0 + lane + 1 == n_bags && e != n_keys))) bad = true;
    e = e < s ? s : (e > n_keys ? n_keys : e);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long x = __shfl_up_sync(0xffffffffu, e, o);
      if (lane >= o && x > e) {
        e = x;
        bad = true;
      }
    }
    // every position must get a (row, bag) pair even when the offsets are
    // malformed: the first bag starts at 0 and the last one ends at n_keys
    if (b0 == 0) s = 0;
    if (lane == nb - 1 && b0 + nb == n_bags) e = n_keys;
    if (lane >= nb) e = LLONG_MAX;
    if (bad) latch(st, kErrInvalid);
    const long long E = __shfl_sync(0xffffffffu, e, nb - 1);
    for (long long ws = s; ws < E; ws += 32) {
      const long long p = ws + lane;
      int cnt = 0;
      for (int j = 0; j < nb; ++j) cnt += (__shfl_sync(0xffffffffu, e, j) <= p);
      if (p < E) {
        const long long k = __ldg(keys + p);
        unsigned r = sentinel;
        if (k < 0) {
          latch(st, kErrInvalid);
        } else {
          const long long off = probe_find(m, (unsigned long long)k);
          if (off < 0)
            latch(st, kErrNotFound);
          else
            r = (unsigned)off;
        }
        rkey[p] = r;
        rval[p] = (unsigned)(b0 + cnt);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// LSD radix sort of 32-bit keys with 32-bit values, 8-bit digits, stable
// ---------------------------------------------------------------------------
constexpr int kRadixThreads = 256;
constexpr int kRadixItems = 16;
constexpr int kRadixWarpItems = 32 * kRadixItems;                     // 512
constexpr int kRadixTile = kRadixWarpItems * (kRadixThreads / 32);    // 4096
constexpr int kRadixBins = 256;

// Per-tile digit counts, stored digit-major: hist[d * ntiles + tile].
// Lanes holding the same digit are merged with match.any before the shared
// counter is bumped, so a hot row costs one atomic per warp round.
__global__ void __launch_bounds__(kRadixThreads)
radix_hist_kernel(const unsigned* __restrict__ keys, long long n, int shift,
                  unsigned* __restrict__ hist, long long ntiles) {
  __shared__ unsigned h[kRadixBins];
  h[threadIdx.x] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const long long base = (long long)blockIdx.x * kRadixTile + (long long)wid * kRadixWarpItems;
#pragma unroll 4
  for (int r = 0; r < kRadixItems; ++r) {
    const long long p = base + r * 32 + lane;
    const unsigned d = p < n ? ((__ldg(keys + p) >> shift) & 255u) : 256u;
    const unsigned peers = __match_any_sync(0xffffffffu, d);
    if (d < 256u && (__ffs(peers) - 1) == lane) atomicAdd(&h[d], (unsigned)__popc(peers));
  }
  __syncthreads();
  hist[(long long)threadIdx.x * ntiles + blockIdx.x] = h[threadIdx.x];
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

// In-place exclusive scan of one digit's row hist[d * ntiles, +ntiles); block
// d also writes the digit total.
__global__ void __launch_bounds__(256)
radix_scan_kernel(unsigned* __restrict__ hist, long long ntiles, unsigned* __restrict__ totals) {
  __shared__ unsigned wsum[8];
  unsigned* row = hist + (long long)blockIdx.x * ntiles;
  unsigned carry = 0;
  for (long long b = 0; b < ntiles; b += 256) {
    const long long i = b + threadIdx.x;
    const unsigned x = i < ntiles ? row[i] : 0u;
    unsigned tot;
    const unsigned ex = block_exclusive_scan_256(x, wsum, tot);
    if (i < ntiles) row[i] = carry + ex;
    carry += tot;
  }
  if (threadIdx.x == 0) totals[blockIdx.x] = carry;
}

// Stable scatter of one tile.  Each warp ranks its 512 items in order (16
// rounds of 32 lanes; match.any gives the rank among equal digits within a
// round, a per-warp shared counter carries it across rounds), the block turns
// per-warp counts into tile-local digit offsets, the items are placed in
// digit order in shared memory and written out in runs, one run per digit,
// to the tile's global offsets.
__global__ void __launch_bounds__(kRadixThreads)
radix_scatter_kernel(const unsigned* __restrict__ kin, const unsigned* __restrict__ vin,
                     unsigned* __restrict__ kout, unsigned* __restrict__ vout, long long n,
                     int shift, const unsigned* __restrict__ hist,
                     const unsigned* __restrict__ totals, long long ntiles) {
  __shared__ unsigned s_k[kRadixTile];
  __shared__ unsigned s_v[kRadixTile];
  __shared__ unsigned wc[8][kRadixBins + 1];
  __shared__ unsigned dstart[kRadixBins];
  __shared__ unsigned gbase[kRadixBins];
  __shared__ unsigned wsum[8];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const long long tile0 = (long long)blockIdx.x * kRadixTile;
  const int tile_n = (int)min((long long)kRadixTile, n - tile0);

  for (int i = threadIdx.x; i < 8 * (kRadixBins + 1); i += kRadixThreads) (&wc[0][0])[i] = 0;
  {
    unsigned tot;
    const unsigned dpre = block_exclusive_scan_256(totals[threadIdx.x], wsum, tot);
    gbase[threadIdx.x] = dpre + hist[(long long)threadIdx.x * ntiles + blockIdx.x];
  }
  __syncthreads();

  unsigned k[kRadixItems], v[kRadixItems], lr[kRadixItems];
  const long long base = tile0 + (long long)wid * kRadixWarpItems;
#pragma unroll
  for (int r = 0; r < kRadixItems; ++r) {
    const long long p = base + r * 32 + lane;
    const bool ok = p < n;
    k[r] = ok ? __ldg(kin + p) : 0u;
    v[r] = ok ? __ldg(vin + p) : 0u;
  }
  const unsigned lt = lanemask_lt();
#pragma unroll
  for (int r = 0; r < kRadixItems; ++r) {
    const long long p = base + r * 32 + lane;
    const unsigned d = p < n ? ((k[r] >> shift) & 255u) : 256u;
    const unsigned peers = __match_any_sync(0xffffffffu, d);
    const unsigned before = wc[wid][d];
    lr[r] = before + __popc(peers & lt);
    __syncwarp();
    if ((__ffs(peers) - 1) == lane) wc[wid][d] = before + __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  {
    const int d = threadIdx.x;
    unsigned pre = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      const unsigned t = wc[w][d];
      wc[w][d] = pre;
      pre += t;
    }
    unsigned tot;
    dstart[d] = block_exclusive_scan_256(pre, wsum, tot);
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kRadixItems; ++r) {
    const long long p = base + r * 32 + lane;
    if (p < n) {
      const unsigned d = (k[r] >> shift) & 255u;
      const unsigned pos = dstart[d] + wc[wid][d] + lr[r];
      s_k[pos] = k[r];
      s_v[pos] = v[r];
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < tile_n; i += kRadixThreads) {
    const unsigned key = s_k[i];
    const unsigned d = (key >> shift) & 255u;
    const unsigned o = gbase[d] + (unsigned)i - dstart[d];
    kout[o] = key;
    vout[o] = s_v[i];
  }
}

#endif  // DHS_TEMPLATES_ONLY

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

// Group of G lanes, lane gl holding float4 columns gl + q*G (q < NV) of the
// row gradient in fp64; rowwise_sq is the fp64 sum of g^2 over the row (only
// used by row-wise Adagrad, computed by the caller over the group).
template <int NV>
__device__ __forceinline__ void update_row_vec(float* row, int dim, int gl, int G,
                                               const double (&acc)[NV][4], const OptArgs& o,
                                               double rowwise_sq) {
  const int d4 = dim >> 2;
  float4* w4 = reinterpret_cast<float4*>(row);
  if (o.opt == 3) {
    // one accumulator per row, stored at row[dim]; every lane computes the
    // same new value, lane 0 stores it
    const float G0 = row[dim];
    const float Gn = __fadd_rn(G0, (float)(rowwise_sq / (double)dim));
    const float den = __fadd_rn(__fsqrt_rn(Gn), o.eps);
#pragma unroll
    for (int q = 0; q < NV; ++q) {
      const int c4 = gl + q * G;
      if (c4 >= d4) continue;
      float4 w = w4[c4];
      float* wp = &w.x;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float g = (float)acc[q][e];
        wp[e] = __fsub_rn(wp[e], __fdiv_rn(__fmul_rn(o.lr, g), den));
      }
      w4[c4] = w;
    }
    if (gl == 0) row[dim] = Gn;
    return;
  }
#pragma unroll
  for (int q = 0; q < NV; ++q) {
    const int c4 = gl + q * G;
    if (c4 >= d4) continue;
    float4 w = w4[c4];
    float* wp = &w.x;
    if (o.opt == 0) {
#pragma unroll
      for (int e = 0; e < 4; ++e) wp[e] = sgd_w(wp[e], (float)acc[q][e], o.lr);
    } else if (o.opt == 1) {
      float4 Gs = w4[d4 + c4];
      float* gp = &Gs.x;
#pragma unroll
      for (int e = 0; e < 4; ++e) adagrad_step(wp[e], gp[e], (float)acc[q][e], o.lr, o.eps);
      w4[d4 + c4] = Gs;
    } else {
      float4 ms = w4[d4 + c4], vs = w4[2 * d4 + c4];
      float *mp = &ms.x, *vp = &vs.x;
#pragma unroll
      for (int e = 0; e < 4; ++e) adam_step(wp[e], mp[e], vp[e], (float)acc[q][e], o);
      w4[d4 + c4] = ms;
      w4[2 * d4 + c4] = vs;
    }
    w4[c4] = w;
  }
}

// Scalar form for one column j (used by the combine kernel).
__device__ __forceinline__ void update_col(float* row, int dim, int j, float g, const OptArgs& o,
                                           float rowwise_den) {
  float w = row[j];
  if (o.opt == 0) {
    w = sgd_w(w, g, o.lr);
  } else if (o.opt == 1) {
    float G = row[dim + j];
    adagrad_step(w, G, g, o.lr, o.eps);
    row[dim + j] = G;
  } else if (o.opt == 2) {
    float m = row[dim + j], v = row[2 * dim + j];
    adam_step(w, m, v, g, o);
    row[dim + j] = m;
    row[2 * dim + j] = v;
  } else {
    w = __fsub_rn(w, __fdiv_rn(__fmul_rn(o.lr, g), rowwise_den));
  }
  row[j] = w;
}

// ---------------------------------------------------------------------------
// segment reduce + update
// ---------------------------------------------------------------------------
enum : unsigned char { kPieceHead = 1, kPieceThrough = 2, kPieceTailStart = 4 };

// A group of G lanes owns sort chunk c = [cC, cC + C).  It sums, in fp64 and
// in sorted (= batch) order, the gradients of every segment that starts in the
// chunk and applies the optimizer to that row once.  A segment that started
// in an earlier chunk is skipped unless it is "long" (spans >= 3 chunks), in
// which case this chunk's piece is written as a partial.  A segment that
// starts here and ends in the next chunk is finished here (short overrun); one
// that reaches chunk c + 2 is long: its piece up to the chunk end is written
// as the starting partial and bwd_combine_kernel finishes it.
template <int G, int NV>
__global__ void __launch_bounds__(256)
bwd_seg_kernel(const unsigned* __restrict__ skey, const unsigned* __restrict__ sval, long long n,
               const float* __restrict__ grad, long long n_bags, int dim, RowSpace rs, OptArgs oa,
               double* __restrict__ part_head, double* __restrict__ part_tail,
               unsigned char* __restrict__ cflags, int C, DevState* st) {
  constexpr int U = G < 8 ? G : 8;
  const int lane = threadIdx.x & 31;
  const int gl = lane & (G - 1);
  const int gw = lane / G;
  const unsigned gmask = (G == 32) ? 0xffffffffu : (((1u << G) - 1u) << (gw * G));
  const long long gid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / G;
  const long long ngroups = ((long long)gridDim.x * blockDim.x) / G;
  const long long nchunks = (n + C - 1) / C;
  const unsigned long long nrows = st->row_count;
  const int d4 = dim >> 2;
  const int pstride = NV * G * 4;  // doubles per partial vector
  unsigned long long nseg_total = 0;

  for (long long c = gid; c < nchunks; c += ngroups) {
    const long long start = c * C;
    const long long end = min(n, start + C);
    unsigned char flags = 0;
    unsigned nseg = 0;

    double acc[NV][4];
#pragma unroll
    for (int q = 0; q < NV; ++q)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[q][e] = 0.0;

    // mode of the piece being read: 0 skip, 1 long head piece, 2 owned short
    // segment, 3 long segment starting here
    int mode;
    unsigned cur = __ldg(skey + start);
    if (start > 0 && __ldg(skey + start - 1) == cur) {
      const bool head_long = (c >= 2 && __ldg(skey + (c - 1) * (long long)C - 1) == cur) ||
                             ((c + 1) * (long long)C < n && __ldg(skey + (c + 1) * (long long)C) == cur);
      mode = head_long ? 1 : 0;
    } else {
      ++nseg;
      mode = ((c + 2) * (long long)C < n && __ldg(skey + (c + 2) * (long long)C) == cur) ? 3 : 2;
    }

    auto close_piece = [&](bool continues) {
      if (mode == 1) {
        double* o = part_head + c * (long long)pstride;
#pragma unroll
        for (int q = 0; q < NV; ++q)
#pragma unroll
          for (int e = 0; e < 4; ++e) o[(q * G + gl) * 4 + e] = acc[q][e];
        flags |= continues ? kPieceThrough : kPieceHead;
      } else if (mode == 3) {
        double* o = part_tail + c * (long long)pstride;
#pragma unroll
        for (int q = 0; q < NV; ++q)
#pragma unroll
          for (int e = 0; e < 4; ++e) o[(q * G + gl) * 4 + e] = acc[q][e];
        flags |= kPieceTailStart;
      } else if (mode == 2 && cur < nrows) {
        double sq = 0.0;
        if (oa.opt == 3) {
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
        update_row_vec<NV>(rs.row(cur), dim, gl, G, acc, oa, sq);
      }
#pragma unroll
      for (int q = 0; q < NV; ++q)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[q][e] = 0.0;
    };

    bool done = false;
    for (long long ws = start; ws < n && !done; ws += G) {
      const int cnt = (int)min((long long)G, n - ws);
      const unsigned kk = gl < cnt ? __ldg(skey + ws + gl) : 0u;
      const unsigned vv = gl < cnt ? __ldg(sval + ws + gl) : 0u;
      for (int t0 = 0; t0 < cnt && !done; t0 += U) {
        float4 x[U][NV];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int t = t0 + u;
          const unsigned bt = __shfl_sync(gmask, vv, t & (G - 1), G);
          const unsigned ktt = __shfl_sync(gmask, kk, t & (G - 1), G);
          const bool ok = t < cnt && bt < n_bags && ktt < nrows;
          const float4* gr = reinterpret_cast<const float4*>(grad + (long long)bt * dim);
#pragma unroll
          for (int q = 0; q < NV; ++q) {
            const int c4 = gl + q * G;
            x[u][q] = (ok && c4 < d4) ? __ldg(gr + c4) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int t = t0 + u;
          if (done || t >= cnt) break;
          const long long p = ws + t;
          const unsigned kt = __shfl_sync(gmask, kk, t & (G - 1), G);
          if (kt != cur) {
            close_piece(false);
            if (p >= end) {
              done = true;
              break;
            }
            cur = kt;
            ++nseg;
            mode = ((c + 2) * (long long)C < n && __ldg(skey + (c + 2) * (long long)C) == cur) ? 3 : 2;
          } else if (p == end && mode != 2) {
            // a long piece (head or starting) stops at the chunk end
            close_piece(true);
            done = true;
            break;
          }
          if (mode != 0) {
#pragma unroll
            for (int q = 0; q < NV; ++q) {
              acc[q][0] += (double)x[u][q].x;
              acc[q][1] += (double)x[u][q].y;
              acc[q][2] += (double)x[u][q].z;
              acc[q][3] += (double)x[u][q].w;
            }
          }
        }
      }
    }
    if (!done) close_piece(false);  // reached the end of the array
    if (gl == 0) {
      cflags[c] = flags;
      if (cur >= nrows && nseg) --nseg;  // the sentinel run is not a row
      nseg_total += nseg;
    }
  }
  if (gl == 0 && nseg_total) atomicAdd(&st->sum_unique, nseg_total);
}

#ifndef DHS_TEMPLATES_ONLY
// One thread block per long segment (chunks flagged kPieceTailStart): find the
// run of partials (through pieces up to the first head piece), sum them in
// fp64 in a fixed order, and apply the optimizer to the row.
__global__ void __launch_bounds__(256)
bwd_combine_kernel(const unsigned* __restrict__ skey, long long n, int dim, RowSpace rs,
                   OptArgs oa, const double* __restrict__ part_head,
                   const double* __restrict__ part_tail, const unsigned char* __restrict__ cflags,
                   int C, int pstride, DevState* st) {
  extern __shared__ double sacc[];  // [slices][dim]
  __shared__ long long s_end;
  __shared__ double s_sq;
  const long long nchunks = (n + C - 1) / C;
  const unsigned long long nrows = st->row_count;
  const int T = blockDim.x;
  const int slices = dim >= T ? 1 : T / dim;
  for (long long c = blockIdx.x; c < nchunks; c += gridDim.x) {
    if (!(cflags[c] & kPieceTailStart)) continue;
    const unsigned key = skey[(c + 1) * (long long)C - 1];
    // the run ends at the first chunk after c whose piece is a head piece
    if (threadIdx.x == 0) s_end = nchunks - 1;
    __syncthreads();
    for (long long b = c + 1; b < nchunks; b += T) {
      const long long k = b + threadIdx.x;
      const bool is_end = k < nchunks && (cflags[k] & kPieceHead);
      const unsigned any = __syncthreads_or(is_end);
      if (is_end) atomicMin((unsigned long long*)&s_end, (unsigned long long)k);
      __syncthreads();
      if (any) break;
    }
    const long long kend = s_end;
    // sums: slice s adds pieces s, s + slices, ... (piece 0 = starting partial)
    const long long npieces = kend - c + 1;
    for (int j0 = 0; j0 < dim; j0 += (slices == 1 ? T : dim)) {
      const int sl = slices == 1 ? 0 : threadIdx.x / dim;
      const int j = slices == 1 ? j0 + threadIdx.x : threadIdx.x % dim;
      if (sl < slices && j < dim) {
        double a = 0.0;
        for (long long pc = sl; pc < npieces; pc += slices) {
          const double* src = pc == 0 ? part_tail + c * (long long)pstride
                                      : part_head + (c + pc) * (long long)pstride;
          a += src[j];
        }
        sacc[sl * dim + j] = a;
      }
      if (slices != 1) break;
    }
    __syncthreads();
    // fold slices in order into slice 0
    if (threadIdx.x < dim || slices == 1) {
      for (int j = threadIdx.x; j < dim && slices > 1; j += T) {
        double a = sacc[j];
        for (int s = 1; s < slices; ++s) a += sacc[s * dim + j];
        sacc[j] = a;
      }
    }
    __syncthreads();
    if (key < nrows) {
      float* row = rs.row(key);
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
        const float Gn = __fadd_rn(row[dim], (float)(s_sq / (double)dim));
        den = __fadd_rn(__fsqrt_rn(Gn), oa.eps);
        __syncthreads();
        if (threadIdx.x == 0) row[dim] = Gn;
      }
      for (int j = threadIdx.x; j < dim; j += T) update_col(row, dim, j, (float)sacc[j], oa, den);
    }
    __syncthreads();
  }
}

#endif  // DHS_TEMPLATES_ONLY

}  // namespace dhs
