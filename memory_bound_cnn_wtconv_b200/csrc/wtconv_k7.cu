// Kernels for k = 7.
#define WTC_K 7
#include "wtconv_kinst.cuh"
