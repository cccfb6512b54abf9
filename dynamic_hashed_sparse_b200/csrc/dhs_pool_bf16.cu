// Forward pool kernels for tables with bf16 weights (dim a multiple of 8 in
// [32, 512]: a lane's 16-byte unit holds 8 weights, so the shapes are those
// of fp32 rows of half the width).
#include "dhs_pool_impl.cuh"

namespace dhs {

cudaError_t launch_probe_pool_bf16(int G, int NV, int sm_count, IdMap m, RowSpace rs, int dim,
                                   const long long* keys, long long n_keys, const long long* bag_off,
                                   long long n_bags, const float* psw, bool mean, float* out, unsigned* nbm,
                                   unsigned* slotpos, int ctr_sel, DevState* st, cudaStream_t s) {
#define DHS_RUN(g, v) \
  pool_impl::run_form<g, v, true>(sm_count, m, rs, dim, keys, n_keys, bag_off, n_bags, psw, mean, out, nbm, slotpos, ctr_sel, st, s)
  switch (G * 100 + NV) {
    case 401: return DHS_RUN(4, 1);
    case 801: return DHS_RUN(8, 1);
    case 1601: return DHS_RUN(16, 1);
    case 3201: return DHS_RUN(32, 1);
    case 3202: return DHS_RUN(32, 2);
  }
#undef DHS_RUN
  return cudaErrorInvalidValue;
}

cudaError_t launch_pool_refs_bf16(int G, int NV, int sm_count, RowSpace rs, int dim, const Slot* slots,
                                  long long* refs, long long n_keys, const long long* bag_off,
                                  long long n_bags, const float* psw, bool mean, float* out, DevState* st,
                                  cudaStream_t s) {
#define DHS_RUN(g, v) \
  pool_impl::run_refs_form<g, v, true>(sm_count, rs, dim, slots, refs, n_keys, bag_off, n_bags, psw, mean, out, st, s)
  switch (G * 100 + NV) {
    case 401: return DHS_RUN(4, 1);
    case 801: return DHS_RUN(8, 1);
    case 1601: return DHS_RUN(16, 1);
    case 3201: return DHS_RUN(32, 1);
    case 3202: return DHS_RUN(32, 2);
  }
#undef DHS_RUN
  return cudaErrorInvalidValue;
}

}  // namespace dhs
