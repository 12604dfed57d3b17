// Single translation unit for libkda.so (one definition of the device status
// word shared by every kernel).
#include "kda_api.cu"
#include "kda_chunk.cu"
#include "kda_dplr.cu"
#include "kda_decode.cu"
#include "kda_backward.cu"
#include "kda_gemm.cu"
#include "kda_layer.cu"
#include "kda_noalloc.cu"
