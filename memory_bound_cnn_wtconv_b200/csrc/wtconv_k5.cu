// Kernels for k = 5.
#define WTC_K 5
#include "wtconv_kinst.cuh"
