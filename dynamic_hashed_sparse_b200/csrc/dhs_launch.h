// Host-side launchers of the width-templated kernels (one translation unit
// each, so that they compile in parallel).
#pragma once

#include <cuda_runtime.h>

#include <utility>

#include "dhs_device.cuh"

namespace dhs {

struct OptArgs;

// Launch of a hot-path kernel (one whose first statement is pdl_enter()):
// with DHS_PDL, as a programmatic dependent of the work before it in the
// stream.  Returns the launch's error.
template <typename... P, typename... A>
cudaError_t launch_k(void (*kernel)(P...), unsigned grid, unsigned block, size_t smem, cudaStream_t s,
                     A&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = DHS_PDL ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

// Blocks of `kernel` (launched with `threads` threads and `smem` bytes of
// dynamic shared memory) that fit on one SM of the current device, at least
// 1.  Looked up once per kernel, device and shared-memory size and cached
// (safe to call from several host threads); a kernel asking for more than
// 48 KB of dynamic shared memory has its limit raised on the device first.
int blocks_per_sm(const void* kernel, int threads, size_t smem);

// fwd_probe_pool_kernel<G, NV, PM>; returns a cudaError_t of the launch.
// psw: per-sample weights (NULL: none); mean: divide each bag by its length.
cudaError_t launch_probe_pool(int G, int NV, int sm_count, IdMap m, RowSpace rs, int dim,
                              const long long* keys, long long n_keys, const long long* bag_off,
                              long long n_bags, const float* psw, bool mean, float* out, unsigned* nbm,
                              unsigned* slotpos, int ctr_sel, DevState* st, cudaStream_t s);

// fwd_pool_refs_kernel<G, NV, PM> (gather + pool from per-id row references)
cudaError_t launch_pool_refs(int G, int NV, int sm_count, RowSpace rs, int dim, const Slot* slots,
                             long long* refs, long long n_keys, const long long* bag_off,
                             long long n_bags, const float* psw, bool mean, float* out, DevState* st,
                             cudaStream_t s);

// the same two for tables with bf16 weights (G, NV from dim / 2)
cudaError_t launch_probe_pool_bf16(int G, int NV, int sm_count, IdMap m, RowSpace rs, int dim,
                                   const long long* keys, long long n_keys, const long long* bag_off,
                                   long long n_bags, const float* psw, bool mean, float* out, unsigned* nbm,
                                   unsigned* slotpos, int ctr_sel, DevState* st, cudaStream_t s);
cudaError_t launch_pool_refs_bf16(int G, int NV, int sm_count, RowSpace rs, int dim, const Slot* slots,
                                  long long* refs, long long n_keys, const long long* bag_off,
                                  long long n_bags, const float* psw, bool mean, float* out, DevState* st,
                                  cudaStream_t s);

// bwd_seg_kernel<G, NV, OPT, EXT>, one entry point per optimizer and pooling
// form (_ext: per-sample weights or mean pooling; bagpos / mult / mean are
// used only there)
#define DHS_SEG_DECL(NAME_)                                                                     \
  cudaError_t NAME_(int G, int NV, int sm_count, const unsigned* skey, const unsigned* sval,    \
                    long long n, const float* grad, long long n_bags, int dim, RowSpace rs,     \
                    const OptArgs& oa, double* part_head, double* part_tail,                    \
                    int chunk, unsigned* chunk_ctr, unsigned* owners, unsigned* owner_ctr,      \
                    DevState* st, const unsigned* bagpos, const double* mult, bool mean,        \
                    const RunTable& rt, cudaStream_t s);
DHS_SEG_DECL(launch_seg_sgd)
DHS_SEG_DECL(launch_seg_adagrad)
DHS_SEG_DECL(launch_seg_adam)
DHS_SEG_DECL(launch_seg_rowwise)
DHS_SEG_DECL(launch_seg_sgd_ext)
DHS_SEG_DECL(launch_seg_adagrad_ext)
DHS_SEG_DECL(launch_seg_adam_ext)
DHS_SEG_DECL(launch_seg_rowwise_ext)
#undef DHS_SEG_DECL

// bwd_segw_kernel<CPL, OPT, EXT, BF> (a warp per chunk, CPL columns per
// lane; bf16: the table's weights are bf16; rt: the arrival table of the
// long segments, or key == nullptr)
#define DHS_SEGW_DECL(NAME_)                                                                    \
  cudaError_t NAME_(int cpl, bool bf16, int sm_count, const unsigned* skey, const unsigned* sval, \
                    long long n, const float* grad, long long n_bags, int dim, RowSpace rs,     \
                    const OptArgs& oa, double* part_head, double* part_tail, int pstride,       \
                    int chunk, unsigned* chunk_ctr, unsigned* owners, unsigned* owner_ctr,      \
                    DevState* st, const unsigned* bagpos, const double* mult, bool mean,        \
                    const RunTable& rt, cudaStream_t s);
DHS_SEGW_DECL(launch_seg_sgd_w)
DHS_SEGW_DECL(launch_seg_adagrad_w)
DHS_SEGW_DECL(launch_seg_adam_w)
DHS_SEGW_DECL(launch_seg_rowwise_w)
DHS_SEGW_DECL(launch_seg_sgd_ext_w)
DHS_SEGW_DECL(launch_seg_adagrad_ext_w)
DHS_SEGW_DECL(launch_seg_adam_ext_w)
DHS_SEGW_DECL(launch_seg_rowwise_ext_w)
#undef DHS_SEGW_DECL

}  // namespace dhs
