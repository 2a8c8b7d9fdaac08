// sgemm.h -- fp32 CUDA-core GEMM used by the absorb (see sgemm.cu).
#pragma once

#include <cuda_runtime.h>

namespace ispa {

// C[M,N] = alpha * op(A)[M,K] * op(B)[K,N] + beta * C, row-major, op = transpose when ta / tb.
cudaError_t sgemm(bool ta, bool tb, int M, int N, int K, float alpha, const float* A, long long lda, const float* B,
                  long long ldb, float beta, float* C, long long ldc, bool lower_only, cudaStream_t s,
                  int* n_launched);

}  // namespace ispa
