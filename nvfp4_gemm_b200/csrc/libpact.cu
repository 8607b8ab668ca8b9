// libpact.cu -- the library is one translation unit (so that the per-device status
// word and the kernels share one module without relocatable device code).
#include "api.cu"
#include "quant.cu"
#include "gemm.cu"
#include "lora.cu"
#include "gptq.cu"
