// bwd_seg_kernel instantiations for row-wise Adagrad.
#include "dhs_seg_impl.cuh"
DHS_SEG_TU(3, launch_seg_rowwise)
