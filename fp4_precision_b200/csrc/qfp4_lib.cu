// qfp4_lib.cu - the library as one translation unit, so that the kernels and
// the entry points share the device error word without relocatable device code.
#include "quant.cu"
#include "gemm_sm100.cu"
#include "qfp4_api.cu"
