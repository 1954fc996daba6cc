// The DyT kernels over bf16 activations (see dyt_select.cuh).
#include "dyt_select_impl.cuh"

DYT_INSTANTIATE_SELECTORS(__nv_bfloat16)
