// bwd_seg_kernel instantiations for SGD.
#include "dhs_seg_impl.cuh"
DHS_SEG_TU(0, launch_seg_sgd)
