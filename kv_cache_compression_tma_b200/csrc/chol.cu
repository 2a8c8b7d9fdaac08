// chol.cu -- diagonal-block kernel of the blocked Cholesky factorisation used by the absorb.
//
// The absorb solves (G + lam I) dW = R W (ISPA summary, section 2, stage 2, closed form).  G + lam I
// is symmetric positive definite for lam > 0, so it is factorised as L L^T by a blocked
// right-looking Cholesky with 128-wide panels; this kernel handles one 128 x 128 diagonal block
// (a smaller last block is padded with the identity, whose factor and inverse are the identity):
//   1. Cholesky of the block, right-looking over four 32-wide sub-blocks:
//        a. one warp factorises the 32 x 32 diagonal sub-block in registers (lane = row, column
//           broadcasts by shuffle, one reciprocal per column),
//        b. one thread per row below it solves its row of the sub-panel (registers),
//        c. all threads apply the rank-32 update to the trailing lower triangle (4 x 4 register tiles);
//      a pivot <= 0 or non-finite sets the NOT_SPD status bit and the kernel stops;
//   2. the inverse X = L^-1 by 2 x 2 block recursion, [[L11, 0], [L21, L22]]^-1 =
//      [[X11, 0], [-X22 L21 X11, X22]]: the four 32 x 32 diagonal inverses by forward substitution
//      (one warp each, lane = column), then the 32 -> 64 level, then the 64 -> 128 level, each
//      off-diagonal block as two small GEMMs (T = L21 X11, X21 = -X22 T),
//      so that the panel solve and the triangular solves of the right-hand side become GEMMs.
// One CTA, 256 threads, fp32 throughout (the factor's storage precision): every step of the
// sequential chains is a register FMA, a shuffle or one reciprocal per column.
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
constexpr size_t kSmem = sizeof(float) * (2 * kB * kLd + (kB / 2) * kLd + kB) + 16;

// Step J of the warp-level Cholesky of a 32 x 32 block held one row per lane (a[k] = row's column
// k): pivot broadcast, column scaling, rank-1 update of the trailing rows.  Template recursion keeps
// every register index a compile-time constant.
template <int J>
__device__ __forceinline__ void warp_potrf_step(float (&a)[kS], int lane, bool& ok) {
  if constexpr (J < kS) {
    const float piv = __shfl_sync(0xffffffffu, a[J], J);
    if (!(piv > 0.f) || !isfinite(piv)) ok = false;
    const float inv = rsqrtf(fmaxf(piv, 1e-30f));
    const float ljj = piv * inv;
    // lanes above the diagonal keep updating their (never stored, never read) upper entries: this
    // keeps the warp convergent and every update unpredicated
    a[J] = lane == J ? ljj : a[J] * inv;
#pragma unroll
    for (int k = J + 1; k < kS; ++k) a[k] = fmaf(-a[J], __shfl_sync(0xffffffffu, a[J], k), a[k]);
    warp_potrf_step<J + 1>(a, lane, ok);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    potrf_trtri_kernel(float* A, long long lda, int nb, float* Linv, unsigned* status) {
  extern __shared__ __align__(16) float sm[];
  float* L = sm;
  float* X = sm + kB * kLd;
  float* T = X + kB * kLd;         // [64][kLd] products L21 X11 of one recursion level
  float* rdiag = T + (kB / 2) * kLd;  // 1 / L_ii
  volatile int* bad = reinterpret_cast<volatile int*>(rdiag + kB);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) *bad = 0;
  {
    // all 64 loads of a thread issued up front; thread t owns column t % 128 of rows t / 128 + 2p,
    // so every warp instruction reads 128 contiguous bytes of one row
    const int j = tid & (kB - 1), i0 = tid >> 7;
    float v[kB / 2];
#pragma unroll
    for (int p = 0; p < kB / 2; ++p) {
      const int i = i0 + 2 * p;
      v[p] = (i < nb && j <= i) ? A[static_cast<long long>(i) * lda + j] : 0.f;
    }
#pragma unroll
    for (int p = 0; p < kB / 2; ++p) {
      const int i = i0 + 2 * p;
      L[i * kLd + j] = (i >= nb && i == j) ? 1.f : v[p];
      X[i * kLd + j] = 0.f;
    }
  }
  __syncthreads();

  // ---------------------------------------------------------------- 1. Cholesky
  for (int kb = 0; kb < kNS; ++kb) {
    const int c0 = kb * kS;
    if (warp == 0) {
      const int row = c0 + lane;
      float a[kS];
#pragma unroll
      for (int k = 0; k < kS; ++k) a[k] = k <= lane ? L[row * kLd + c0 + k] : 0.f;
      bool ok = true;
      warp_potrf_step<0>(a, lane, ok);
      if (!ok && lane == 0) *bad = 1;
#pragma unroll
      for (int k = 0; k < kS; ++k)
        if (k <= lane) L[row * kLd + c0 + k] = a[k];
      __syncwarp();
      rdiag[row] = 1.f / L[row * kLd + row];
    }
    __syncthreads();
    if (*bad) break;
    const int r0 = c0 + kS, n2 = kB - r0;
    if (tid < n2) {
      const int r = r0 + tid;
      float x[kS];
#pragma unroll
      for (int k = 0; k < kS; ++k) x[k] = L[r * kLd + c0 + k];
#pragma unroll
      for (int k = 0; k < kS; ++k) {
        float s = x[k];
#pragma unroll
        for (int j = 0; j < k; ++j) s = fmaf(-x[j], L[(c0 + k) * kLd + c0 + j], s);
        x[k] = s * rdiag[c0 + k];
      }
#pragma unroll
      for (int k = 0; k < kS; ++k) L[r * kLd + c0 + k] = x[k];
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
    float x[kS];
#pragma unroll
    for (int i = 0; i < kS; ++i) {
      float s = (i == c) ? 1.f : 0.f;
#pragma unroll
      for (int j = 0; j < i; ++j) s = fmaf(-L[(c0 + i) * kLd + c0 + j], x[j], s);
      x[i] = s * rdiag[c0 + i];
    }
#pragma unroll
    for (int i = 0; i < kS; ++i) X[(c0 + i) * kLd + c0 + c] = x[i];
  }
  __syncthreads();
  // recursion levels: blocks of size h = 32 (two pairs) then h = 64 (one pair).  For a pair whose
  // lower-left h x h block sits at rows i0.., columns j0.. (i0 = j0 + h):
  //   T = L[i0.., j0..] X[j0.., j0..]   then   X[i0.., j0..] = -X[i0.., i0..] T
  // T holds pair pr's h x h block at columns pr*h (row stride kLd); every thread owns 4 (h=32) or
  // 16 (h=64) outputs in a 2 x 2 / 4 x 4 register tile.
  for (int h = kS; h < kB; h *= 2) {
    const int npairs = kB / (2 * h);
    const int tiles_per_pair = (h / 2) * (h / 2) / (h == kS ? 1 : 4);  // threads per pair
    const int tw = h == kS ? 2 : 4;                                   // register tile width
    for (int pass = 0; pass < 2; ++pass) {
      for (int e = tid; e < npairs * tiles_per_pair; e += kThreads) {
        const int pr = e / tiles_per_pair, tix = e % tiles_per_pair;
        const int j0 = pr * 2 * h, i0 = j0 + h;
        const int nt = h / tw;
        const int rr = (tix / nt) * tw, cc = (tix % nt) * tw;
        float acc[4][4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) acc[u][v] = 0.f;
        // pass 0: T = L21 X11 (inner dimension over the X11 rows j0..j0+h)
        // pass 1: X21 = -X22 T (inner dimension over the X22 columns i0..i0+h)
        const float* Am = pass == 0 ? L + (i0 + rr) * kLd + j0 : X + (i0 + rr) * kLd + i0;
        const float* Bm = pass == 0 ? X + j0 * kLd + j0 + cc : T + pr * h + cc;
        for (int k = 0; k < h; ++k) {
          float av[4], bv[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            av[u] = u < tw ? Am[u * kLd + k] : 0.f;
            bv[u] = u < tw ? Bm[k * kLd + u] : 0.f;
          }
#pragma unroll
          for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(av[u], bv[v], acc[u][v]);
        }
        float* out = pass == 0 ? T + rr * kLd + pr * h + cc : X + (i0 + rr) * kLd + j0 + cc;
        const float sgn = pass == 0 ? 1.f : -1.f;
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v)
            if (u < tw && v < tw) out[u * kLd + v] = sgn * acc[u][v];
      }
      __syncthreads();
    }
  }

  // ---------------------------------------------------------------- 3. factor and inverse out
  {
    const int j = tid & (kB - 1), i0 = tid >> 7;
#pragma unroll 8
    for (int p = 0; p < kB / 2; ++p) {
      const int i = i0 + 2 * p;
      if (i < nb && j < nb) A[static_cast<long long>(i) * lda + j] = j <= i ? L[i * kLd + j] : 0.f;
      Linv[i * kB + j] = (i < nb && j < nb) ? X[i * kLd + j] : 0.f;
    }
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
