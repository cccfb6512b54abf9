// bwd_seg_kernel instantiations for Adagrad (per-element accumulator).
#include "dhs_seg_impl.cuh"
DHS_SEG_TU(1, launch_seg_adagrad)
