// libmacaq.cu -- the library's single translation unit (kernels share the device status
// flag, so they are compiled together rather than with relocatable device code).
#include "api.cu"
#include "quant.cu"
#include "flip.cu"
#include "gemm.cu"
#include "noalloc.cu"
#include "calib.cu"
