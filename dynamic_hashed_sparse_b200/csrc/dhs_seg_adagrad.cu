// Segment-kernel instantiations for Adagrad (per-element accumulator), sum pooling.
#include "dhs_seg_impl.cuh"
DHS_SEG_TU(1, false, launch_seg_adagrad)
