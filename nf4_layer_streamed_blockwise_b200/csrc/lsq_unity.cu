// Single translation unit of the lsq library (one device module, so every
// kernel sees the same device status word without relocatable device code).
#include "abi.cu"
#include "nf4_quant.cu"
#include "gemm_tc.cu"
#include "gemm_nf4.cu"
#include "lora_grad.cu"
#include "layer_ops.cu"
#include "attention_tc.cu"
#include "attention.cu"
#include "stream.cu"
#include "noalloc.cu"
