// Host-side launchers of the width-templated kernels (one translation unit
// each, so that they compile in parallel).
#pragma once

#include <cuda_runtime.h>

#include "dhs_device.cuh"

namespace dhs {

struct OptArgs;

// fwd_probe_pool_kernel<G, NV>; returns a cudaError_t of the launch.
cudaError_t launch_probe_pool(int G, int NV, int sm_count, IdMap m, RowSpace rs, int dim,
                              const long long* keys, long long n_keys, const long long* bag_off,
                              long long n_bags, float* out, unsigned* nbm, unsigned* slotpos,
                              DevState* st, cudaStream_t s);

// fwd_pool_refs_kernel<G, NV> (gather + pool from per-id row references)
cudaError_t launch_pool_refs(int G, int NV, int sm_count, RowSpace rs, int dim, const Slot* slots,
                             const long long* refs, long long n_keys, const long long* bag_off,
                             long long n_bags, float* out, DevState* st, cudaStream_t s);

// bwd_seg_kernel<G, NV, OPT>, one entry point per optimizer
#define DHS_SEG_DECL(NAME_)                                                                     \
  cudaError_t NAME_(int G, int NV, int sm_count, const unsigned* skey, const unsigned* sval,    \
                    long long n, const float* grad, long long n_bags, int dim, RowSpace rs,     \
                    const OptArgs& oa, double* part_head, double* part_tail,                    \
                    int chunk, unsigned* chunk_ctr, unsigned* owners, unsigned* owner_ctr,      \
                    DevState* st, cudaStream_t s);
DHS_SEG_DECL(launch_seg_sgd)
DHS_SEG_DECL(launch_seg_adagrad)
DHS_SEG_DECL(launch_seg_adam)
DHS_SEG_DECL(launch_seg_rowwise)
#undef DHS_SEG_DECL

// bwd_segw_kernel<CPL, OPT> (a warp per chunk, CPL columns per lane)
#define DHS_SEGW_DECL(NAME_)                                                                    \
  cudaError_t NAME_(int cpl, int sm_count, const unsigned* skey, const unsigned* sval,         \
                    long long n, const float* grad, long long n_bags, int dim, RowSpace rs,     \
                    const OptArgs& oa, double* part_head, double* part_tail, int pstride,       \
                    int chunk, unsigned* chunk_ctr, unsigned* owners, unsigned* owner_ctr,      \
                    DevState* st, cudaStream_t s);
DHS_SEGW_DECL(launch_seg_sgd_w)
DHS_SEGW_DECL(launch_seg_adagrad_w)
DHS_SEGW_DECL(launch_seg_adam_w)
DHS_SEGW_DECL(launch_seg_rowwise_w)
#undef DHS_SEGW_DECL

}  // namespace dhs
