// Single translation unit of the library: the device status word is shared
// by every kernel without relocatable device code.
#include "api.cu"
#include "gemm.cu"
#include "permute.cu"
#include "quant.cu"
#include "swiglu_bwd.cu"
#include "transpose.cu"
#include "noalloc.cu"
#include "router.cu"
#include "scales.cu"
