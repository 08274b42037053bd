// tm_lib.cu -- single translation unit of libtm.so (the device error word and all
// kernels live in one module, so no relocatable device code is needed).
#include "tm_kernels.cu"
#include "tm_backward.cu"
#include "tm_gemm.cu"
#include "tm_api.cu"
#include "tm_profile.cu"
#include "tm_noalloc.cu"
