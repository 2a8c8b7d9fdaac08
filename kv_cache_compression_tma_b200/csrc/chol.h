// chol.h -- diagonal-block Cholesky + triangular inverse (see chol.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace ispa {

// Reads the nb x nb (nb <= 128) lower block at A (row stride lda, a multiple of 4; nb a multiple of
// 4), adds *shift (device fp64, may be null) to its diagonal, computes the Cholesky factor L of the
// result and writes L^-1 into Linv (128 x 128, row stride 128, zero outside nb x nb).  A is not
// written; entries above its diagonal are never used.  Sets the NOT_SPD status bit on a
// non-positive pivot and then leaves Linv unwritten.  pdl: launch with programmatic stream
// serialisation (the first read of A waits for the previous grid of the stream).
cudaError_t potrf_trtri(const float* A, long long lda, int nb, const double* shift, float* Linv, unsigned* status,
                        cudaStream_t s, int* n_launched, bool pdl = false);

}  // namespace ispa
