// Single translation unit of libactsparse: the device status word and every
// kernel live in one module, so no relocatable device code is needed.
#include "weight_prep.cu"
#include "select.cu"
#include "decode.cu"
#include "gemm.cu"
#include "fp8.cu"
#include "rsparse.cu"
#include "rsparse_prefill.cu"
#include "hybrid.cu"
#include "abi.cu"
#include "noalloc.cu"
