// The DyT kernels over f16 activations (see dyt_select.cuh).
#include "dyt_select_impl.cuh"

DYT_INSTANTIATE_SELECTORS(__half)
