// chol.cu -- diagonal-block kernel of the blocked Cholesky factorisation used by the absorb.
//
// The absorb solves (G + lam I) dW = R W (ISPA summary, section 2, stage 2, closed form).  G + lam I
// is symmetric positive definite for lam > 0, so it is factorised as L L^T by a blocked
// right-looking Cholesky with 128-wide panels; this kernel handles one diagonal block:
//   1. unblocked Cholesky of the block in fp64 shared memory (a pivot <= 0 or non-finite sets the
//      NOT_SPD status bit and the block is left unchanged),
//   2. the explicit inverse of the block's triangular factor, so that the panel solve and the
//      triangular solves of the right-hand side become plain GEMMs.
// One CTA, 256 threads.
#include <math.h>

#include "chol.h"
#include "internal.h"
#include "sm100.cuh"

namespace ispa {
namespace {

constexpr int kB = 128;
constexpr int kLd = kB + 1;
constexpr int kThreads = 256;
constexpr size_t kSmem = sizeof(double) * kB * kLd + sizeof(float) * kB * kLd + 16;

__global__ void __launch_bounds__(kThreads, 1)
    potrf_trtri_kernel(float* A, long long lda, int nb, float* Linv, unsigned* status) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  double* L = reinterpret_cast<double*>(smem_raw);
  float* X = reinterpret_cast<float*>(smem_raw + sizeof(double) * kB * kLd);
  volatile int* bad = reinterpret_cast<volatile int*>(smem_raw + sizeof(double) * kB * kLd + sizeof(float) * kB * kLd);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) *bad = 0;
  for (int idx = tid; idx < kB * kB; idx += kThreads) {
    const int i = idx / kB, j = idx % kB;
    L[i * kLd + j] = (i < nb && j <= i) ? static_cast<double>(A[static_cast<long long>(i) * lda + j]) : 0.0;
  }
  __syncthreads();
  for (int j = 0; j < nb; ++j) {
    if (tid == 0) {
      const double piv = L[j * kLd + j];
      if (!(piv > 0.0) || !isfinite(piv))
        *bad = 1;
      else
        L[j * kLd + j] = sqrt(piv);
    }
    __syncthreads();
    if (*bad) break;
    const double inv = 1.0 / L[j * kLd + j];
    for (int i = j + 1 + tid; i < nb; i += kThreads) L[i * kLd + j] *= inv;
    __syncthreads();
    for (int i = j + 1 + warp; i < nb; i += kThreads / 32) {
      const double lij = L[i * kLd + j];
      for (int k = j + 1 + lane; k <= i; k += 32) L[i * kLd + k] -= lij * L[k * kLd + j];
    }
    __syncthreads();
  }
  if (*bad) {
    if (tid == 0) atomicOr(status, kStatusNotSpd);
    return;
  }
  // factor back to global (lower triangle; strict upper of the diagonal block cleared)
  for (int idx = tid; idx < nb * nb; idx += kThreads) {
    const int i = idx / nb, j = idx % nb;
    A[static_cast<long long>(i) * lda + j] = j <= i ? static_cast<float>(L[i * kLd + j]) : 0.f;
  }
  // inverse of the triangular factor, one column per thread: L x = e_c by forward substitution
  const int c = tid;
  if (c < kB) {
    for (int i = 0; i < kB; ++i) X[i * kLd + c] = 0.f;
  }
  for (int i = 0; i < nb; ++i) {
    if (c < nb && c <= i) {
      double s = (i == c) ? 1.0 : 0.0;
      for (int j = c; j < i; ++j) s -= L[i * kLd + j] * static_cast<double>(X[j * kLd + c]);
      X[i * kLd + c] = static_cast<float>(s / L[i * kLd + i]);
    }
  }
  __syncthreads();
  for (int idx = tid; idx < kB * kB; idx += kThreads) {
    const int i = idx / kB, j = idx % kB;
    Linv[idx] = (i < nb && j < nb) ? X[i * kLd + j] : 0.f;
  }
}

}  // namespace

cudaError_t potrf_trtri(float* A, long long lda, int nb, float* Linv, unsigned* status, cudaStream_t s,
                        int* n_launched) {
  cudaError_t e = cudaFuncSetAttribute(potrf_trtri_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmem));
  if (e != cudaSuccess) return e;
  potrf_trtri_kernel<<<1, kThreads, kSmem, s>>>(A, lda, nb, Linv, status);
  *n_launched += 1;
  return cudaGetLastError();
}

}  // namespace ispa
