// Segment-kernel instantiations for Adam, per-sample weights or mean pooling.
#include "dhs_seg_impl.cuh"
DHS_SEG_TU(2, true, launch_seg_adam_ext)
