// Segment-kernel instantiations for row-wise Adagrad, sum pooling.
#include "dhs_seg_impl.cuh"
DHS_SEG_TU(3, false, launch_seg_rowwise)
