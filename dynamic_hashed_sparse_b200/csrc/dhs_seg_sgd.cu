// Segment-kernel instantiations for SGD, sum pooling.
#include "dhs_seg_impl.cuh"
DHS_SEG_TU(0, false, launch_seg_sgd)
