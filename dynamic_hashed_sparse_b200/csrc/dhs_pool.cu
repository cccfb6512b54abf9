// Instantiations of the fused probe + gather + pool kernel and of the
// gather + pool from row references, for each row width.
#include <algorithm>

#define DHS_TEMPLATES_ONLY

#include "dhs_fwd.cuh"
#include "dhs_launch.h"

namespace dhs {

namespace {
template <int G, int NV>
cudaError_t run(int sm_count, IdMap m, RowSpace rs, int dim, const long long* keys,
                long long n_keys, const long long* bag_off, long long n_bags, float* out,
                unsigned* nbm, unsigned* slotpos, DevState* st, cudaStream_t s) {
  static int resident = 0;
  if (!resident) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fwd_probe_pool_kernel<G, NV>,
                                                      kFwdThreads, 0) != cudaSuccess || per_sm < 1) {
      cudaGetLastError();
      per_sm = 1;
    }
    resident = per_sm * sm_count;
  }
  const long long nchunks = (n_bags + G - 1) / G;
  const long long per_block = kFwdThreads / G;
  const long long need = std::max<long long>(1, (nchunks + per_block - 1) / per_block);
  const long long grid = std::min<long long>(need, resident);
  fwd_probe_pool_kernel<G, NV><<<(unsigned)grid, kFwdThreads, 0, s>>>(
      m, rs, dim, keys, n_keys, bag_off, n_bags, out, nbm, slotpos, st);
  return cudaGetLastError();
}

template <int G, int NV>
cudaError_t run_refs(int sm_count, RowSpace rs, int dim, const Slot* slots, const long long* refs,
                     long long n_keys, const long long* bag_off, long long n_bags, float* out,
                     DevState* st, cudaStream_t s) {
  static int resident = 0;
  if (!resident) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fwd_pool_refs_kernel<G, NV>, kFwdThreads, 0) !=
            cudaSuccess || per_sm < 1) {
      cudaGetLastError();
      per_sm = 1;
    }
    resident = per_sm * sm_count;
  }
  const long long nchunks = (n_bags + G - 1) / G;
  const long long per_block = kFwdThreads / G;
  const long long need = std::max<long long>(1, (nchunks + per_block - 1) / per_block);
  const long long grid = std::min<long long>(need, resident);
  fwd_pool_refs_kernel<G, NV><<<(unsigned)grid, kFwdThreads, 0, s>>>(rs, dim, slots, refs, n_keys, bag_off,
                                                                      n_bags, out, st);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_probe_pool(int G, int NV, int sm_count, IdMap m, RowSpace rs, int dim,
                              const long long* keys, long long n_keys, const long long* bag_off,
                              long long n_bags, float* out, unsigned* nbm, unsigned* slotpos,
                              DevState* st, cudaStream_t s) {
#define DHS_RUN(g, v) run<g, v>(sm_count, m, rs, dim, keys, n_keys, bag_off, n_bags, out, nbm, slotpos, st, s)
  switch (G * 100 + NV) {
    case 101: return DHS_RUN(1, 1);
    case 201: return DHS_RUN(2, 1);
    case 401: return DHS_RUN(4, 1);
    case 801: return DHS_RUN(8, 1);
    case 1601: return DHS_RUN(16, 1);
    case 3201: return DHS_RUN(32, 1);
    case 3202: return DHS_RUN(32, 2);
    case 3204: return DHS_RUN(32, 4);
  }
#undef DHS_RUN
  return cudaErrorInvalidValue;
}

cudaError_t launch_pool_refs(int G, int NV, int sm_count, RowSpace rs, int dim, const Slot* slots,
                             const long long* refs, long long n_keys, const long long* bag_off,
                             long long n_bags, float* out, DevState* st, cudaStream_t s) {
#define DHS_RUN(g, v) run_refs<g, v>(sm_count, rs, dim, slots, refs, n_keys, bag_off, n_bags, out, st, s)
  switch (G * 100 + NV) {
    case 101: return DHS_RUN(1, 1);
    case 201: return DHS_RUN(2, 1);
    case 401: return DHS_RUN(4, 1);
    case 801: return DHS_RUN(8, 1);
    case 1601: return DHS_RUN(16, 1);
    case 3201: return DHS_RUN(32, 1);
    case 3202: return DHS_RUN(32, 2);
    case 3204: return DHS_RUN(32, 4);
  }
#undef DHS_RUN
  return cudaErrorInvalidValue;
}

}  // namespace dhs
