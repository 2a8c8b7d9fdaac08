// sgemm.cu -- fp32 GEMM on CUDA cores: C = alpha * op(A) op(B) + beta * C (the absorb when d % 128 != 0, the fp32 projection).
//
// Row-major operands with leading dimensions; op(X) = X or X^T.  128 x 128 output tile per block,
// 256 threads with an 8 x 8 register micro-tile, K in steps of 8 double-buffered through shared
// memory.  `lower_only` skips tiles strictly above the diagonal (symmetric rank-k updates of the
// Cholesky trailing matrix touch only its lower triangle).
//
// In-place use is allowed in exactly one pattern, which the absorb relies on: when the output
// block covers all of one operand's rows that feed it (M <= 128 with C aliasing B, or N <= 128
// with C aliasing A), every block reads its whole input panel before its epilogue writes the same
// panel, and no other block touches it.
#include "internal.h"
#include "sgemm.h"

namespace ispa {
namespace {

constexpr int kBM = 128, kBN = 128, kBK = 8, kPad = 4;

template <bool TA, bool TB>
__global__ void __launch_bounds__(256) sgemm_kernel(int M, int N, int K, float alpha, const float* A, long long lda,
                                                    const float* B, long long ldb, float beta, float* C,
                                                    long long ldc, int lower_only) {
  __shared__ __align__(16) float As[2][kBK][kBM + kPad];
  __shared__ __align__(16) float Bs[2][kBK][kBN + kPad];
  const int tid = threadIdx.x;
  const int m0 = blockIdx.y * kBM, n0 = blockIdx.x * kBN;
  if (lower_only && n0 > m0 + kBM - 1) return;
  const int ty = tid >> 4, tx = tid & 15;

  float ra[4], rb[4];
  auto load = [&](int k0) {
    if (!TA) {
      const int i = tid >> 1, kq = (tid & 1) * 4;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int k = k0 + kq + q;
        ra[q] = (m0 + i < M && k < K) ? A[static_cast<long long>(m0 + i) * lda + k] : 0.f;
      }
    } else {
      const int k = tid >> 5, iq = (tid & 31) * 4;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = m0 + iq + q;
        ra[q] = (i < M && k0 + k < K) ? A[static_cast<long long>(k0 + k) * lda + i] : 0.f;
      }
    }
    if (!TB) {
      const int k = tid >> 5, jq = (tid & 31) * 4;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int j = n0 + jq + q;
        rb[q] = (k0 + k < K && j < N) ? B[static_cast<long long>(k0 + k) * ldb + j] : 0.f;
      }
    } else {
      const int j = tid >> 1, kq = (tid & 1) * 4;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int k = k0 + kq + q;
        rb[q] = (n0 + j < N && k < K) ? B[static_cast<long long>(n0 + j) * ldb + k] : 0.f;
      }
    }
  };
  auto store = [&](int buf) {
    if (!TA) {
      const int i = tid >> 1, kq = (tid & 1) * 4;
#pragma unroll
      for (int q = 0; q < 4; ++q) As[buf][kq + q][i] = ra[q];
    } else {
      const int k = tid >> 5, iq = (tid & 31) * 4;
#pragma unroll
      for (int q = 0; q < 4; ++q) As[buf][k][iq + q] = ra[q];
    }
    if (!TB) {
      const int k = tid >> 5, jq = (tid & 31) * 4;
#pragma unroll
      for (int q = 0; q < 4; ++q) Bs[buf][k][jq + q] = rb[q];
    } else {
      const int j = tid >> 1, kq = (tid & 1) * 4;
#pragma unroll
      for (int q = 0; q < 4; ++q) Bs[buf][kq + q][j] = rb[q];
    }
  };

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  const int nk = (K + kBK - 1) / kBK;
  load(0);
  store(0);
  __syncthreads();
  for (int kt = 0; kt < nk; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < nk) load((kt + 1) * kBK);
#pragma unroll
    for (int k = 0; k < kBK; ++k) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][k][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][k][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][k][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][k][64 + tx * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    if (kt + 1 < nk) store(buf ^ 1);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (r >= M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
      if (c >= N) continue;
      float* p = C + static_cast<long long>(r) * ldc + c;
      *p = beta == 0.f ? alpha * acc[i][j] : fmaf(alpha, acc[i][j], beta * *p);
    }
  }
}

}  // namespace

cudaError_t sgemm(bool ta, bool tb, int M, int N, int K, float alpha, const float* A, long long lda, const float* B,
                  long long ldb, float beta, float* C, long long ldc, bool lower_only, cudaStream_t s,
                  int* n_launched) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  dim3 grid((N + kBN - 1) / kBN, (M + kBM - 1) / kBM);
  const int lo = lower_only ? 1 : 0;
  if (!ta && !tb)
    sgemm_kernel<false, false><<<grid, 256, 0, s>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, lo);
  else if (!ta && tb)
    sgemm_kernel<false, true><<<grid, 256, 0, s>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, lo);
  else if (ta && !tb)
    sgemm_kernel<true, false><<<grid, 256, 0, s>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, lo);
  else
    sgemm_kernel<true, true><<<grid, 256, 0, s>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, lo);
  *n_launched += 1;
  return cudaGetLastError();
}

}  // namespace ispa
