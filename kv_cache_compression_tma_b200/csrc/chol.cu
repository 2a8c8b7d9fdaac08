// chol.cu -- diagonal-block kernel of the blocked Cholesky factorisation used by the absorb.
//
// The absorb solves (G + lam I) dW = R W (ISPA summary, section 2, stage 2, closed form).  G + lam I
// is symmetric positive definite for lam > 0, so it is factorised as L L^T by a blocked
// right-looking Cholesky with 128-wide panels; this kernel handles one 128 x 128 diagonal block
// (a smaller last block is padded with the identity, whose factor and inverse are the identity):
//   1. Cholesky of the block, right-looking over four 32-wide sub-blocks:
//        a. one warp factorises the 32 x 32 diagonal sub-block in fp64 registers (lane = row,
//           column broadcasts by shuffle),
//        b. one thread per row below it solves its row of the sub-panel (fp64 registers),
//        c. all threads apply the rank-32 update to the trailing lower triangle (4 x 4 register tiles);
//      a pivot <= 0 or non-finite sets the NOT_SPD status bit and the kernel stops;
//   2. the inverse X = L^-1: the four diagonal sub-blocks by forward substitution (one warp each,
//      lane = column), then the off-diagonal sub-blocks by distance from the diagonal:
//        X_ij = -X_ii * sum_{k=j}^{i-1} L_ik X_kj,
//      so that the panel solve and the triangular solves of the right-hand side become GEMMs.
// One CTA, 256 threads, shared memory holds L and X in fp32 (the factor's storage precision).
#include <math.h>

#include "chol.h"
#include "internal.h"
#include "sm100.cuh"

namespace ispa {
namespace {

constexpr int kB = 128;   // block size
constexpr int kS = 32;    // sub-block size
constexpr int kNS = kB / kS;
constexpr int kLd = kB + 1;
constexpr int kThreads = 256;
constexpr size_t kSmem = sizeof(float) * (2 * kB * kLd + (kNS - 1) * kS * (kS + 1)) + 16;

__global__ void __launch_bounds__(kThreads, 1)
    potrf_trtri_kernel(float* A, long long lda, int nb, float* Linv, unsigned* status) {
  extern __shared__ __align__(16) float sm[];
  float* L = sm;
  float* X = sm + kB * kLd;
  float* T = X + kB * kLd;  // [kNS-1][kS][kS+1] products of one distance level
  volatile int* bad = reinterpret_cast<volatile int*>(T + (kNS - 1) * kS * (kS + 1));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const unsigned full = 0xffffffffu;

  if (tid == 0) *bad = 0;
  for (int idx = tid; idx < kB * kB; idx += kThreads) {
    const int i = idx / kB, j = idx % kB;
    float v = 0.f;
    if (i < nb && j < nb)
      v = j <= i ? A[static_cast<long long>(i) * lda + j] : 0.f;
    else if (i == j)
      v = 1.f;
    L[i * kLd + j] = v;
    X[i * kLd + j] = 0.f;
  }
  __syncthreads();

  // ---------------------------------------------------------------- 1. Cholesky
  for (int kb = 0; kb < kNS; ++kb) {
    const int c0 = kb * kS;
    if (warp == 0) {
      const int row = c0 + lane;
      double a[kS];
#pragma unroll
      for (int k = 0; k < kS; ++k) a[k] = k <= lane ? static_cast<double>(L[row * kLd + c0 + k]) : 0.0;
      bool ok = true;
#pragma unroll
      for (int j = 0; j < kS; ++j) {
        const double piv = __shfl_sync(full, a[j], j);
        if (!(piv > 0.0) || !isfinite(piv)) ok = false;
        const double ljj = sqrt(fmax(piv, 1e-300));
        if (lane == j) a[j] = ljj;
        if (lane > j) a[j] = a[j] / ljj;
#pragma unroll
        for (int k = j + 1; k < kS; ++k) {
          const double lkj = __shfl_sync(full, a[j], k);
          if (lane >= k) a[k] -= a[j] * lkj;
        }
      }
      if (!ok && lane == 0) *bad = 1;
#pragma unroll
      for (int k = 0; k < kS; ++k)
        if (k <= lane) L[row * kLd + c0 + k] = static_cast<float>(a[k]);
    }
    __syncthreads();
    if (*bad) break;
    const int r0 = c0 + kS, n2 = kB - r0;
    if (tid < n2) {
      const int r = r0 + tid;
      double x[kS];
#pragma unroll
      for (int k = 0; k < kS; ++k) x[k] = L[r * kLd + c0 + k];
#pragma unroll
      for (int k = 0; k < kS; ++k) {
        double s = x[k];
#pragma unroll
        for (int j = 0; j < k; ++j) s -= x[j] * static_cast<double>(L[(c0 + k) * kLd + c0 + j]);
        x[k] = s / static_cast<double>(L[(c0 + k) * kLd + c0 + k]);
      }
#pragma unroll
      for (int k = 0; k < kS; ++k) L[r * kLd + c0 + k] = static_cast<float>(x[k]);
    }
    __syncthreads();
    if (n2 > 0) {
      const int nt = n2 / 4;
      for (int t = tid; t < nt * nt; t += kThreads) {
        const int ti = t / nt, tj = t % nt;
        if (tj > ti) continue;
        const int i0 = r0 + 4 * ti, j0 = r0 + 4 * tj;
        float acc[4][4];
#pragma unroll
        for (int p = 0; p < 4; ++p)
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[p][q] = 0.f;
#pragma unroll 8
        for (int k = 0; k < kS; ++k) {
          float ai[4], aj[4];
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            ai[p] = L[(i0 + p) * kLd + c0 + k];
            aj[p] = L[(j0 + p) * kLd + c0 + k];
          }
#pragma unroll
          for (int p = 0; p < 4; ++p)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[p][q] = fmaf(ai[p], aj[q], acc[p][q]);
        }
#pragma unroll
        for (int p = 0; p < 4; ++p)
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (j0 + q <= i0 + p) L[(i0 + p) * kLd + j0 + q] -= acc[p][q];
      }
    }
    __syncthreads();
  }
  if (*bad) {
    if (tid == 0) atomicOr(status, kStatusNotSpd);
    return;
  }

  // ---------------------------------------------------------------- 2. inverse of the factor
  if (warp < kNS) {
    const int c0 = warp * kS, c = lane;
    double x[kS];
#pragma unroll
    for (int i = 0; i < kS; ++i) {
      double s = (i == c) ? 1.0 : 0.0;
#pragma unroll
      for (int j = 0; j < i; ++j) s -= static_cast<double>(L[(c0 + i) * kLd + c0 + j]) * x[j];
      x[i] = s / static_cast<double>(L[(c0 + i) * kLd + c0 + i]);
    }
#pragma unroll
    for (int i = 0; i < kS; ++i) X[(c0 + i) * kLd + c0 + c] = static_cast<float>(x[i]);
  }
  __syncthreads();
  for (int dist = 1; dist < kNS; ++dist) {
    const int nblk = kNS - dist;
    for (int e = tid; e < nblk * kS * kS; e += kThreads) {
      const int b = e / (kS * kS), r = (e / kS) % kS, c = e % kS;
      const int bi = b + dist, bj = b;
      double s = 0.0;
      for (int k = kS * bj; k < kS * bi; ++k)
        s += static_cast<double>(L[(kS * bi + r) * kLd + k]) * X[k * kLd + kS * bj + c];
      T[(b * kS + r) * (kS + 1) + c] = static_cast<float>(s);
    }
    __syncthreads();
    for (int e = tid; e < nblk * kS * kS; e += kThreads) {
      const int b = e / (kS * kS), r = (e / kS) % kS, c = e % kS;
      const int bi = b + dist, bj = b;
      double s = 0.0;
#pragma unroll 8
      for (int m = 0; m < kS; ++m)
        s += static_cast<double>(X[(kS * bi + r) * kLd + kS * bi + m]) * T[(b * kS + m) * (kS + 1) + c];
      X[(kS * bi + r) * kLd + kS * bj + c] = static_cast<float>(-s);
    }
    __syncthreads();
  }

  // ---------------------------------------------------------------- 3. factor and inverse out
  for (int idx = tid; idx < nb * nb; idx += kThreads) {
    const int i = idx / nb, j = idx % nb;
    A[static_cast<long long>(i) * lda + j] = j <= i ? L[i * kLd + j] : 0.f;
  }
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
