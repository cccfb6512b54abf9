// Segment-kernel instantiations for Adam, sum pooling.
#include "dhs_seg_impl.cuh"
DHS_SEG_TU(2, false, launch_seg_adam)
