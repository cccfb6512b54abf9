// Segment-kernel instantiations for row-wise Adagrad, per-sample weights or mean pooling.
#include "dhs_seg_impl.cuh"
DHS_SEG_TU(3, true, launch_seg_rowwise_ext)
