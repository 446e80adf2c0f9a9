// Kernels for k = 3.
#define WTC_K 3
#include "wtconv_kinst.cuh"
