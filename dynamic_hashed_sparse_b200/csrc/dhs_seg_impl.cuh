// Launchers of the segment kernels for one optimizer and one pooling form
// (EXT: per-sample weights or mean pooling); included by one translation unit
// per (optimizer, form) so that they compile in parallel.
#pragma once

#include <algorithm>

#define DHS_TEMPLATES_ONLY
#include "dhs_bwd.cuh"
#include "dhs_launch.h"

namespace dhs {
namespace seg_impl {

template <int G, int NV, int OPT, bool EXT>
cudaError_t run(int sm_count, const unsigned* skey, const unsigned* sval, long long n,
                const float* grad, long long n_bags, int dim, RowSpace rs, const OptArgs& oa,
                double* part_head, double* part_tail, int chunk,
                unsigned* chunk_ctr, unsigned* owners, unsigned* owner_ctr, DevState* st,
                const unsigned* bagpos, const double* mult, bool mean, const RunTable& rt, cudaStream_t s) {
  const size_t smem = seg_smem_bytes(G, NV);
  const int resident = blocks_per_sm((const void*)bwd_seg_kernel<G, NV, OPT, EXT>, 256, smem) * sm_count;
  const long long nchunks = (n + chunk - 1) / chunk;
  const long long per_block = 256 / G;
  const long long need = std::max<long long>(1, (nchunks + per_block - 1) / per_block);
  const long long grid = std::min<long long>(need, resident);
  launch_k(bwd_seg_kernel<G, NV, OPT, EXT>, (unsigned)grid, 256, smem, s, skey, sval, n, grad, n_bags, dim, rs, oa,
                                                                   part_head, part_tail, chunk, chunk_ctr,
                                                                   owners, owner_ctr, st, bagpos, mult, mean, rt);
  return cudaGetLastError();
}

template <int OPT, bool EXT>
cudaError_t launch(int G, int NV, int sm_count, const unsigned* skey, const unsigned* sval,
                   long long n, const float* grad, long long n_bags, int dim, RowSpace rs,
                   const OptArgs& oa, double* part_head, double* part_tail,
                   int chunk, unsigned* chunk_ctr, unsigned* owners, unsigned* owner_ctr, DevState* st,
                   const unsigned* bagpos, const double* mult, bool mean, const RunTable& rt, cudaStream_t s) {
#define DHS_RUN(g, v)                                                                                \
  run<g, v, OPT, EXT>(sm_count, skey, sval, n, grad, n_bags, dim, rs, oa, part_head, part_tail, chunk, \
                      chunk_ctr, owners, owner_ctr, st, bagpos, mult, mean, rt, s)
  switch (G * 100 + NV) {
    case 102: return DHS_RUN(1, 2);
    case 202: return DHS_RUN(2, 2);
    case 402: return DHS_RUN(4, 2);
    case 802: return DHS_RUN(8, 2);
    case 1602: return DHS_RUN(16, 2);
    case 3202: return DHS_RUN(32, 2);
    case 3204: return DHS_RUN(32, 4);
  }
#undef DHS_RUN
  return cudaErrorInvalidValue;
}

template <int CPL, int OPT, bool EXT, bool BF>
cudaError_t run_w(int sm_count, const unsigned* skey, const unsigned* sval, long long n,
                  const float* grad, long long n_bags, int dim, RowSpace rs, const OptArgs& oa,
                  double* part_head, double* part_tail, int pstride, int chunk, unsigned* chunk_ctr,
                  unsigned* owners, unsigned* owner_ctr, DevState* st, const unsigned* bagpos,
                  const double* mult, bool mean, const RunTable& rt, cudaStream_t s) {
  const size_t smem = segw_smem_bytes(CPL);
  const int resident = blocks_per_sm((const void*)bwd_segw_kernel<CPL, OPT, EXT, BF>, 256, smem) * sm_count;
  const long long nchunks = (n + chunk - 1) / chunk;
  const long long need = std::max<long long>(1, (nchunks + 7) / 8);  // a warp per chunk
  const long long grid = std::min<long long>(need, resident);
  // gradient rows read about once per call (about one id per bag) are marked
  // first to evict in L2
  const bool grad_once = DHS_SEGW_EVICT_FIRST && 2 * n <= 3 * n_bags;
  launch_k(bwd_segw_kernel<CPL, OPT, EXT, BF>, (unsigned)grid, 256, smem, s, skey, sval, n, grad, n_bags, dim, rs, oa,
                                                                  part_head, part_tail, pstride, chunk,
                                                                  chunk_ctr, owners, owner_ctr, st, grad_once,
                                                                  bagpos, mult, mean, rt);
  return cudaGetLastError();
}

template <int OPT, bool EXT>
cudaError_t launch_w(int cpl, bool bf16, int sm_count, const unsigned* skey, const unsigned* sval, long long n,
                     const float* grad, long long n_bags, int dim, RowSpace rs, const OptArgs& oa,
                     double* part_head, double* part_tail, int pstride, int chunk, unsigned* chunk_ctr,
                     unsigned* owners, unsigned* owner_ctr, DevState* st, const unsigned* bagpos,
                     const double* mult, bool mean, const RunTable& rt, cudaStream_t s) {
#define DHS_RUN(c)                                                                                       \
  (bf16 ? run_w<c, OPT, EXT, true>(sm_count, skey, sval, n, grad, n_bags, dim, rs, oa, part_head, part_tail,  \
                                   pstride, chunk, chunk_ctr, owners, owner_ctr, st, bagpos, mult, mean, rt, s) \
        : run_w<c, OPT, EXT, false>(sm_count, skey, sval, n, grad, n_bags, dim, rs, oa, part_head, part_tail, \
                                    pstride, chunk, chunk_ctr, owners, owner_ctr, st, bagpos, mult, mean, rt, s))
  switch (cpl) {
    case 1: return DHS_RUN(1);
    case 2: return DHS_RUN(2);
    case 4: return DHS_RUN(4);
    case 8: return DHS_RUN(8);
    case 16: return DHS_RUN(16);
  }
#undef DHS_RUN
  return cudaErrorInvalidValue;
}

}  // namespace seg_impl
}  // namespace dhs

#define DHS_SEG_TU(OPT_, EXT_, NAME_)                                                           \
  namespace dhs {                                                                               \
  cudaError_t NAME_(int G, int NV, int sm_count, const unsigned* skey, const unsigned* sval,    \
                    long long n, const float* grad, long long n_bags, int dim, RowSpace rs,     \
                    const OptArgs& oa, double* part_head, double* part_tail,                    \
                    int chunk, unsigned* chunk_ctr, unsigned* owners, unsigned* owner_ctr,      \
                    DevState* st, const unsigned* bagpos, const double* mult, bool mean,        \
                    const RunTable& rt, cudaStream_t s) {                                       \
    return seg_impl::launch<OPT_, EXT_>(G, NV, sm_count, skey, sval, n, grad, n_bags, dim, rs, oa, \
                                        part_head, part_tail, chunk, chunk_ctr, owners, owner_ctr, \
                                        st, bagpos, mult, mean, rt, s);                         \
  }                                                                                             \
  cudaError_t NAME_##_w(int cpl, bool bf16, int sm_count, const unsigned* skey, const unsigned* sval, \
                        long long n, const float* grad, long long n_bags, int dim, RowSpace rs,  \
                        const OptArgs& oa, double* part_head, double* part_tail, int pstride,    \
                        int chunk, unsigned* chunk_ctr, unsigned* owners, unsigned* owner_ctr,   \
                        DevState* st, const unsigned* bagpos, const double* mult, bool mean,    \
                        const RunTable& rt, cudaStream_t s) {                                   \
    return seg_impl::launch_w<OPT_, EXT_>(cpl, bf16, sm_count, skey, sval, n, grad, n_bags, dim, rs, oa, \
                                          part_head, part_tail, pstride, chunk, chunk_ctr, owners, \
                                          owner_ctr, st, bagpos, mult, mean, rt, s);            \
  }                                                                                             \
  }
