// Kernels for k = 1.
#define WTC_K 1
#include "wtconv_kinst.cuh"
