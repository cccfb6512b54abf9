// Segment-kernel instantiations for SGD, per-sample weights or mean pooling.
#include "dhs_seg_impl.cuh"
DHS_SEG_TU(0, true, launch_seg_sgd_ext)
