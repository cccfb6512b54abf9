// Segment-kernel instantiations for Adagrad (per-element accumulator), per-sample weights or mean pooling.
#include "dhs_seg_impl.cuh"
DHS_SEG_TU(1, true, launch_seg_adagrad_ext)
