// bwd_seg_kernel instantiations for Adam.
#include "dhs_seg_impl.cuh"
DHS_SEG_TU(2, launch_seg_adam)
