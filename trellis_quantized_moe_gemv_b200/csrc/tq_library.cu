// Single translation unit of libtrellis_moe.so: the components share the device flag
// word and a few launch helpers without relocatable device code.
#include "tq_abi.cu"
#include "tq_route.cu"
#include "tq_hadamard.cu"
#include "tq_decode.cu"
#include "tq_gemv.cu"
#include "tq_gemm.cu"
#include "tq_noalloc.cu"
#include "tq_encode.cu"
