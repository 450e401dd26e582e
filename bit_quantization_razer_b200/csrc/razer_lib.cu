// Single translation unit of librazer.so (keeps the device status word and
// every kernel in one module without relocatable device code).
#include <type_traits>

#include "api.cu"
#include "quantize.cu"
#include "ablation.cu"
#include "dequant.cu"
#include "gemv.cu"
#include "gemv_tma.cu"
#include "variant_decode.cu"
#include "gemm.cu"
#include "gemv_noalloc.cu"
