// Launchers of the fused probe + gather + pool kernel and of the gather +
// pool from row references, for each row width, pooling form (sum, weighted
// sum, mean) and weight storage; included by one translation unit per
// storage type so that they compile in parallel.
#pragma once

#include <algorithm>

#define DHS_TEMPLATES_ONLY

#include "dhs_fwd.cuh"
#include "dhs_launch.h"

namespace dhs {
namespace pool_impl {

template <int G, int NV, int PM, bool BF>
cudaError_t run(int sm_count, IdMap m, RowSpace rs, int dim, const long long* keys,
                long long n_keys, const long long* bag_off, long long n_bags, const float* psw,
                float* out, unsigned* nbm, unsigned* slotpos, int ctr_sel, DevState* st, cudaStream_t s) {
  const int resident =
      blocks_per_sm((const void*)fwd_probe_pool_kernel<G, NV, PM, BF>, kFwdThreads, 0) * sm_count;
  const long long nchunks = (n_bags + G - 1) / G;
  const long long per_block = kFwdThreads / G;
  const long long need = std::max<long long>(1, (nchunks + per_block - 1) / per_block);
  const long long grid = std::min<long long>(need, resident);
  launch_k(fwd_probe_pool_kernel<G, NV, PM, BF>, (unsigned)grid, kFwdThreads, 0, s, 
      m, rs, dim, keys, n_keys, bag_off, n_bags, psw, out, nbm, slotpos, ctr_sel, st);
  return cudaGetLastError();
}

template <int G, int NV, int PM, bool BF>
cudaError_t run_refs(int sm_count, RowSpace rs, int dim, const Slot* slots, long long* refs,
                     long long n_keys, const long long* bag_off, long long n_bags, const float* psw,
                     float* out, DevState* st, cudaStream_t s) {
  const int resident =
      blocks_per_sm((const void*)fwd_pool_refs_kernel<G, NV, PM, BF>, kFwdThreads, 0) * sm_count;
  const long long nchunks = (n_bags + G - 1) / G;
  const long long per_block = kFwdThreads / G;
  const long long need = std::max<long long>(1, (nchunks + per_block - 1) / per_block);
  const long long grid = std::min<long long>(need, resident);
  launch_k(fwd_pool_refs_kernel<G, NV, PM, BF>, (unsigned)grid, kFwdThreads, 0, s, rs, dim, slots, refs, n_keys,
                                                                             bag_off, n_bags, psw, out, st);
  return cudaGetLastError();
}

// the pooling form: 1 weighted sum, 2 mean, 0 plain sum
template <int G, int NV, bool BF>
cudaError_t run_form(int sm_count, IdMap m, RowSpace rs, int dim, const long long* keys, long long n_keys,
                     const long long* bag_off, long long n_bags, const float* psw, bool mean, float* out,
                     unsigned* nbm, unsigned* slotpos, int ctr_sel, DevState* st, cudaStream_t s) {
  if (psw) return run<G, NV, 1, BF>(sm_count, m, rs, dim, keys, n_keys, bag_off, n_bags, psw, out, nbm, slotpos, ctr_sel, st, s);
  if (mean) return run<G, NV, 2, BF>(sm_count, m, rs, dim, keys, n_keys, bag_off, n_bags, psw, out, nbm, slotpos, ctr_sel, st, s);
  return run<G, NV, 0, BF>(sm_count, m, rs, dim, keys, n_keys, bag_off, n_bags, psw, out, nbm, slotpos, ctr_sel, st, s);
}

template <int G, int NV, bool BF>
cudaError_t run_refs_form(int sm_count, RowSpace rs, int dim, const Slot* slots, long long* refs,
                          long long n_keys, const long long* bag_off, long long n_bags, const float* psw,
                          bool mean, float* out, DevState* st, cudaStream_t s) {
  if (psw) return run_refs<G, NV, 1, BF>(sm_count, rs, dim, slots, refs, n_keys, bag_off, n_bags, psw, out, st, s);
  if (mean) return run_refs<G, NV, 2, BF>(sm_count, rs, dim, slots, refs, n_keys, bag_off, n_bags, psw, out, st, s);
  return run_refs<G, NV, 0, BF>(sm_count, rs, dim, slots, refs, n_keys, bag_off, n_bags, psw, out, st, s);
}

}  // namespace pool_impl
}  // namespace dhs
