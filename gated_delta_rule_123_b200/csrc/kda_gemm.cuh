// Interface of the layer's projection GEMM (kda_gemm.cu).
#pragma once

#include "kda_common.cuh"

namespace kda {

// Epilogue of one GEMM launch: what is done with each fp32 accumulator c.
struct GemmEpilogue {
    enum Kind { kStoreBf16 = 0, kNegSoftplus = 1, kNormGate = 2 };
    int kind = kStoreBf16;
    // kStoreBf16: C = bf16(c); when beta_out is set, columns [beta_col0, beta_col0 + H)
    // are also written as beta_out[row * H + (col - beta_col0)] = sigmoid(c) in fp32.
    float* beta_out = nullptr;
    int beta_col0 = 0, H = 0;
    // kNegSoftplus: C = -softplus(c) in fp32 (C's row stride in fp32 elements).
    // kNormGate: C = bf16(o * rsqrt(mean_head(o^2) + 1e-5) * norm_w * sigmoid(c)), with o
    // fp32 [M][ldo] and each 128-column head of the row normalised on its own.
    const float* o_in = nullptr;
    int ldo = 0;
    const float* norm_w = nullptr;
};

// C[M, N] (row stride ldc) = A[M, K] (row stride lda) * W[N, K]^T (row stride ldw):
// bf16 operands, fp32 accumulation on the tensor cores, then the epilogue.
int launch_gemm(const void* A, int lda, const void* W, int ldw, void* C, int ldc, int M, int N, int K,
                const GemmEpilogue& ep, cudaStream_t stream, const char** why);

}  // namespace kda
