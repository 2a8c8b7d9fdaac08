// stats_simt.cu -- warmup sufficient statistics G, R, S on CUDA cores (fp32 accumulation).
//
// Same quantities as the tensor-core kernel (ISPA summary, section 2, stage 2: the factors
// A_loc^T A_loc and A_loc^T (A_full - A_loc) of the closed form, plus D^T D), for fp32 inputs and
// widths the tensor-core kernel does not take.  32 x 32 output tile per block, rows of X staged
// through shared memory 32 at a time; D = A_full - A_loc is formed in fp32 when the second input
// is A_full.
#include "internal.h"
#include "sm100.cuh"

namespace ispa {
namespace {

constexpr int kT = 32;

template <typename T>
__device__ __forceinline__ float ldv(const T* p);
template <>
__device__ __forceinline__ float ldv<float>(const float* p) {
  return *p;
}
template <>
__device__ __forceinline__ float ldv<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

template <typename T>
__global__ void __launch_bounds__(kT * 8) stats_simt_kernel(const T* __restrict__ xl, const T* __restrict__ x2,
                                                            long long m, int d, long long lda, int second_is_full,
                                                            int zero, float* G, float* R, float* S) {
  __shared__ float li[kT][kT + 1], di[kT][kT + 1], lj[kT][kT + 1], dj[kT][kT + 1];
  const int which = blockIdx.z;
  const int i0 = blockIdx.y * kT, j0 = blockIdx.x * kT;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8 threads, 4 outputs each
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (long long r0 = 0; r0 < m; r0 += kT) {
    for (int rr = ty; rr < kT; rr += 8) {
      const long long r = r0 + rr;
      float a_i = 0.f, b_i = 0.f, a_j = 0.f, b_j = 0.f;
      if (r < m) {
        if (i0 + tx < d) {
          a_i = ldv(xl + r * lda + i0 + tx);
          b_i = ldv(x2 + r * lda + i0 + tx);
          if (second_is_full) b_i -= a_i;
        }
        if (j0 + tx < d) {
          a_j = ldv(xl + r * lda + j0 + tx);
          b_j = ldv(x2 + r * lda + j0 + tx);
          if (second_is_full) b_j -= a_j;
        }
      }
      li[rr][tx] = a_i;
      di[rr][tx] = b_i;
      lj[rr][tx] = a_j;
      dj[rr][tx] = b_j;
    }
    __syncthreads();
    for (int rr = 0; rr < kT; ++rr) {
      const float bj = which == 0 ? lj[rr][tx] : dj[rr][tx];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = ty * 4 + q;
        const float ai = which == 2 ? di[rr][i] : li[rr][i];
        acc[q] = fmaf(ai, bj, acc[q]);
      }
    }
    __syncthreads();
  }
  float* out = which == 0 ? G : (which == 1 ? R : S);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int i = i0 + ty * 4 + q, j = j0 + tx;
    if (i < d && j < d) {
      float* o = out + static_cast<long long>(i) * d + j;
      *o = zero ? acc[q] : *o + acc[q];
    }
  }
}

}  // namespace

cudaError_t launch_stats_simt(const StatsLaunch& a, cudaStream_t s, int* n_launched) {
  dim3 grid((a.d + kT - 1) / kT, (a.d + kT - 1) / kT, 3);
  if (a.dtype == 1)
    stats_simt_kernel<float><<<grid, kT * 8, 0, s>>>(reinterpret_cast<const float*>(a.a_loc),
                                                     reinterpret_cast<const float*>(a.a_second), a.m, a.d, a.lda,
                                                     a.second_is_full, a.zero, a.G, a.R, a.S);
  else
    stats_simt_kernel<__nv_bfloat16><<<grid, kT * 8, 0, s>>>(
        reinterpret_cast<const __nv_bfloat16*>(a.a_loc), reinterpret_cast<const __nv_bfloat16*>(a.a_second), a.m,
        a.d, a.lda, a.second_is_full, a.zero, a.G, a.R, a.S);
  *n_launched += 1;
  return cudaGetLastError();
}

}  // namespace ispa
