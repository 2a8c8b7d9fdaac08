// chol.cu -- diagonal-block kernel of the blocked Cholesky factorisation used by the absorb.
//
// The absorb solves (G + lam I) dW = R W (ISPA summary, section 2, stage 2, closed form).  G + lam I
// is symmetric positive definite for lam > 0, so it is factorised as L L^T by a blocked
// right-looking Cholesky with 128-wide panels.  This kernel takes one 128 x 128 diagonal block A
// (already updated by the earlier panels, without the ridge shift: lam is added to its diagonal on
// load, which commutes with the earlier updates; a smaller last block is padded with the identity) and
// writes X = L^-1, the inverse of its Cholesky factor: the panel solve and both triangular solves
// of the right-hand side then run as GEMMs against X.  The factor itself is not written back: the
// callers never read the factor's diagonal blocks, only the panels below them and X.
//
// Inside the block the factorisation is right-looking over four 32-wide sub-blocks k = 0..3:
//   A_k  one warp factorises the 32 x 32 diagonal sub-block and inverts its factor in the same
//        pass (lane = row of the factor, lane = column of the inverse; every step of the chain is
//        a shuffle, one reciprocal and register FMAs), while the other seven warps build the
//        off-diagonal blocks of X that the finished sub-blocks allow, by the block forward
//        substitution X_ij = -X_ii (sum_{m=j..i-1} L_im X_mj);
//   B_k  all warps solve the sub-panel below it, L_rk = A_rk X_kk^T;
//   C_k  all warps apply the rank-32 update A_rc -= L_rk L_ck^T to the trailing lower triangle.
// After the last sub-block all warps finish the bottom block row of X.  A pivot <= 0 or
// non-finite sets the NOT_SPD status bit and the kernel stops without writing X.
//
// Shared memory (fp32, 16-byte aligned rows so that every operand moves as float4):
//   W   128 x 132  the block being factorised; a sub-block of X replaces each dead sub-block of it
//   Lt  128 x 132  the factor's off-diagonal sub-blocks, transposed (Lt[col][row] = L[row][col])
//   Xdt 4 x 32 x 36  the diagonal sub-blocks of X, transposed
//   P   5 x 32 x 36  partial sums of the forward substitution
//   col 2 x 32  the pivot column of the current diagonal sub-block step (broadcast buffer)
// One CTA of 256 threads, fp32 throughout (the factor's storage precision).
#include <math.h>

#include "chol.h"
#include "internal.h"
#include "sm100.cuh"

namespace ispa {
namespace {

constexpr int kB = 128;   // block size
constexpr int kS = 32;    // sub-block size
constexpr int kNS = kB / kS;
constexpr int kLd = 132;  // row stride of W and Lt
constexpr int kLs = 36;   // row stride of the 32 x 32 scratch blocks
constexpr int kThreads = 256;
constexpr int kNP = 5;   // partial-sum slots
constexpr size_t kSmem = sizeof(float) * (2 * kB * kLd + (kNS + kNP) * kS * kLs + 2 * kS) + 16;

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void st4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ float comp(const float4& v, int q) {
  return q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w;
}
// MUFU approximations (relative error about one ulp); the correctly rounded reciprocal costs about
// a hundred cycles more per pivot on the sequential chain
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rsqrt_approx(float x) {
  float y;
  asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Step J of the fused Cholesky + inverse of a 32 x 32 block.  Lane i holds row i of the working
// matrix in a[] (entries right of the diagonal are never read) and column i of the inverse in x[].
// With p the pivot and c_k = a_kJ (k > J) the column below it, the factor's column is c / sqrt(p);
// the trailing rows lose c_i c_k / p, and forward substitution for the inverse's column takes
// x_k -= c_k x_J / p before x_J is scaled by 1 / sqrt(p).  The column reaches every lane through a
// 32-float shared-memory buffer (one store per lane, then float4 broadcast loads), two buffers used
// alternately so that step J + 2 writes only after every lane has passed step J + 1's __syncwarp;
// per step this is one store and at most eight loads instead of up to 32 shuffles.
template <int J>
__device__ __forceinline__ void chol_inv_step(float (&a)[kS], float (&x)[kS], bool& ok, float* colbuf, int lane) {
  if constexpr (J < kS) {
    float* cb = colbuf + (J & 1) * kS;
    cb[lane] = a[J];
    __syncwarp();
    float c[kS];
#pragma unroll
    for (int q = J / 4; q < kS / 4; ++q) {
      const float4 t = ld4(cb + 4 * q);
      c[4 * q] = t.x;
      c[4 * q + 1] = t.y;
      c[4 * q + 2] = t.z;
      c[4 * q + 3] = t.w;
    }
    const float p = c[J];  // pivot, clamped to >= 1e-30 below
    ok = ok && (p > 0.f) && isfinite(p);
    const float pc = fmaxf(p, 1e-30f);
    const float r = rcp_approx(pc);
    const float t = a[J] * r, v = x[J] * r;
#pragma unroll
    for (int k = J + 1; k < kS; ++k) {
      a[k] = fmaf(-t, c[k], a[k]);
      x[k] = fmaf(-c[k], v, x[k]);
    }
    x[J] *= rsqrt_approx(pc);
    chol_inv_step<J + 1>(a, x, ok, colbuf, lane);
  }
}

// One warp's share of a 32 x 32 product: acc[u][v] += sum_kk At[kk][RPL*rg + u] * B[kk][4*cg + v]
// with rg = lane / 8, cg = lane % 8 (the warp covers 4*RPL rows and all 32 columns).  At is the
// left operand stored transposed, so that both operands move as float2/float4 rows.
template <int RPL>
__device__ __forceinline__ void gl_acc(float (&acc)[RPL][4], const float* At, int lda, const float* B, int ldb,
                                       int lane) {
  const float* ap = At + RPL * (lane >> 3);
  const float* bp = B + 4 * (lane & 7);
#pragma unroll 8
  for (int kk = 0; kk < kS; ++kk) {
    float av[RPL];
    if constexpr (RPL == 2) {
      const float2 t = *reinterpret_cast<const float2*>(ap + kk * lda);
      av[0] = t.x;
      av[1] = t.y;
    } else {
#pragma unroll
      for (int q = 0; q < RPL / 4; ++q) {
        const float4 t = ld4(ap + kk * lda + 4 * q);
        av[4 * q] = t.x;
        av[4 * q + 1] = t.y;
        av[4 * q + 2] = t.z;
        av[4 * q + 3] = t.w;
      }
    }
    const float4 b = ld4(bp + kk * ldb);
#pragma unroll
    for (int u = 0; u < RPL; ++u) {
      acc[u][0] = fmaf(av[u], b.x, acc[u][0]);
      acc[u][1] = fmaf(av[u], b.y, acc[u][1]);
      acc[u][2] = fmaf(av[u], b.z, acc[u][2]);
      acc[u][3] = fmaf(av[u], b.w, acc[u][3]);
    }
  }
}

struct Term {
  const float* at;
  int lda;
  const float* b;
  int ldb;
};

// Rows [row_lo, row_lo + 4*RPL) of C = alpha * sum_t op(At_t) B_t (ACC: C += ...), all 32
// columns, one warp.
template <int RPL, int NT, bool ACC = false>
__device__ __forceinline__ void gl_sum(const Term (&t)[NT], int row_lo, float alpha, float* C, int ldc, int lane) {
  float acc[RPL][4];
#pragma unroll
  for (int u = 0; u < RPL; ++u) acc[u][0] = acc[u][1] = acc[u][2] = acc[u][3] = 0.f;
#pragma unroll
  for (int i = 0; i < NT; ++i) gl_acc<RPL>(acc, t[i].at + row_lo, t[i].lda, t[i].b, t[i].ldb, lane);
  float* cp = C + (row_lo + RPL * (lane >> 3)) * ldc + 4 * (lane & 7);
#pragma unroll
  for (int u = 0; u < RPL; ++u) {
    float4 o = make_float4(alpha * acc[u][0], alpha * acc[u][1], alpha * acc[u][2], alpha * acc[u][3]);
    if constexpr (ACC) {
      const float4 c = ld4(cp + u * ldc);
      o.x += c.x;
      o.y += c.y;
      o.z += c.z;
      o.w += c.w;
    }
    st4(cp + u * ldc, o);
  }
}

__device__ __forceinline__ void inv_warps_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kThreads - 32) : "memory"); }

__global__ void __launch_bounds__(kThreads, 1)
    potrf_trtri_kernel(const float* __restrict__ A, long long lda, int nb, const double* __restrict__ shift,
                       float* __restrict__ Linv, unsigned* status) {
  extern __shared__ __align__(16) float sm[];
  float* W = sm;
  float* Lt = W + kB * kLd;
  float* Xdt = Lt + kB * kLd;
  float* P = Xdt + kNS * kS * kLs;
  float* colbuf = P + kNP * kS * kLs;  // 2 x 32: the pivot column of a diagonal sub-block step
  volatile int* bad = reinterpret_cast<volatile int*>(colbuf + 2 * kS);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  griddep_launch_dependents();

  // sub-block views (32 x 32): transposed factor block L_im (i > m), row-major X_mj, transposed
  // X_ii, partial-sum slot s
  auto Lblk_t = [&](int i, int m) -> const float* { return Lt + kS * m * kLd + kS * i; };
  auto Xblk = [&](int m, int j) { return W + kS * m * kLd + kS * j; };
  auto Xdiag_t = [&](int i) { return Xdt + i * kS * kLs; };
  auto Pslot = [&](int s) { return P + s * kS * kLs; };

  if (tid == 0) *bad = 0;
  griddep_wait();  // A is written by the previous grid of the stream (PDL launches)
  {
    // lower triangle of the block as float4 chunks: thread t owns chunk column t % 32 of rows
    // t / 32 + 8p; the diagonal gains the shift; rows and columns past nb hold the identity
    const int c4 = tid & 31, i0 = tid >> 5;
    const float lam = shift ? static_cast<float>(*shift) : 0.f;
    float4 v[kB / 8];
#pragma unroll
    for (int p = 0; p < kB / 8; ++p) {
      const int i = i0 + 8 * p, j = 4 * c4;
      v[p] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < nb && j < nb && j <= i) v[p] = ld4(A + static_cast<long long>(i) * lda + j);
    }
#pragma unroll
    for (int p = 0; p < kB / 8; ++p) {
      const int i = i0 + 8 * p, j = 4 * c4;
      float4 w = v[p];
      if (i - j == 0) w.x += lam;
      if (i - j == 1) w.y += lam;
      if (i - j == 2) w.z += lam;
      if (i - j == 3) w.w += lam;
      if (i >= nb || j >= nb) {
        w.x = (i == j) ? 1.f : 0.f;
        w.y = (i == j + 1) ? 1.f : 0.f;
        w.z = (i == j + 2) ? 1.f : 0.f;
        w.w = (i == j + 3) ? 1.f : 0.f;
      }
      if (j <= i) st4(W + i * kLd + j, w);
    }
  }
  __syncthreads();

  for (int k = 0; k < kNS; ++k) {
    const int c0 = k * kS;
    // ------------------------------------------------------------ A_k
    if (warp == 0) {
      float a[kS], x[kS];
      const float* row = W + (c0 + lane) * kLd + c0;
#pragma unroll
      for (int q = 0; q < kS / 4; ++q) {
        const float4 t = ld4(row + 4 * q);
        a[4 * q] = t.x;
        a[4 * q + 1] = t.y;
        a[4 * q + 2] = t.z;
        a[4 * q + 3] = t.w;
      }
#pragma unroll
      for (int i = 0; i < kS; ++i) x[i] = (i == lane) ? 1.f : 0.f;
      bool ok = true;
      chol_inv_step<0>(a, x, ok, colbuf, lane);
      if (!__all_sync(0xffffffffu, ok) && lane == 0) *bad = 1;
      // X_kk row-major into its own (now dead) sub-block of W, and transposed into Xdt[k]
      float* xw = W + c0 * kLd + c0 + lane;
#pragma unroll
      for (int i = 0; i < kS; ++i) xw[i * kLd] = x[i];
      float* xt = Xdiag_t(k) + lane * kLs;
#pragma unroll
      for (int q = 0; q < kS / 4; ++q) st4(xt + 4 * q, make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]));
    } else {
      // block forward substitution for X, as far as the finished sub-blocks allow (warps 1..7);
      // each partial sum P_ij = sum_m L_im X_mj is accumulated as soon as its terms exist
      const int iw = warp - 1;
      // slots: 0 P_10 then P_32, 1 P_20, 2 P_30, 3 P_21, 4 P_31 (16-row halves as work items)
      if (k == 1) {
        if (iw < 6) {  // P_(o+1)0 = L_(o+1)0 X_00
          const int o = iw >> 1, h = iw & 1;
          const Term t[1] = {{Lblk_t(o + 1, 0), kLd, Xblk(0, 0), kLd}};
          gl_sum<4, 1>(t, 16 * h, 1.f, Pslot(o), kLs, lane);
        }
      } else if (k == 2) {
        if (iw < 4) {  // X_10 = -X_11 P_10
          const Term t[1] = {{Xdiag_t(1), kLs, Pslot(0), kLs}};
          gl_sum<2, 1>(t, 8 * iw, -1.f, Xblk(1, 0), kLd, lane);
        }
        inv_warps_sync();
        for (int it = iw; it < 8; it += 7) {
          const int o = it >> 1, h = it & 1;
          if (o == 0) {  // P_20 += L_21 X_10
            const Term t[1] = {{Lblk_t(2, 1), kLd, Xblk(1, 0), kLd}};
            gl_sum<4, 1, true>(t, 16 * h, 1.f, Pslot(1), kLs, lane);
          } else if (o == 1) {  // P_30 += L_31 X_10
            const Term t[1] = {{Lblk_t(3, 1), kLd, Xblk(1, 0), kLd}};
            gl_sum<4, 1, true>(t, 16 * h, 1.f, Pslot(2), kLs, lane);
          } else if (o == 2) {  // P_21 = L_21 X_11
            const Term t[1] = {{Lblk_t(2, 1), kLd, Xblk(1, 1), kLd}};
            gl_sum<4, 1>(t, 16 * h, 1.f, Pslot(3), kLs, lane);
          } else {  // P_31 = L_31 X_11
            const Term t[1] = {{Lblk_t(3, 1), kLd, Xblk(1, 1), kLd}};
            gl_sum<4, 1>(t, 16 * h, 1.f, Pslot(4), kLs, lane);
          }
        }
      } else if (k == 3) {
        if (iw < 4) {  // X_20 = -X_22 P_20, X_21 = -X_22 P_21
          const int o = iw >> 1, h = iw & 1;
          const Term t[1] = {{Xdiag_t(2), kLs, Pslot(o == 0 ? 1 : 3), kLs}};
          gl_sum<4, 1>(t, 16 * h, -1.f, Xblk(2, o), kLd, lane);
        }
        inv_warps_sync();
        if (iw < 6) {
          const int o = iw >> 1, h = iw & 1;
          if (o == 0) {  // P_30 += L_32 X_20
            const Term t[1] = {{Lblk_t(3, 2), kLd, Xblk(2, 0), kLd}};
            gl_sum<4, 1, true>(t, 16 * h, 1.f, Pslot(2), kLs, lane);
          } else if (o == 1) {  // P_31 += L_32 X_21
            const Term t[1] = {{Lblk_t(3, 2), kLd, Xblk(2, 1), kLd}};
            gl_sum<4, 1, true>(t, 16 * h, 1.f, Pslot(4), kLs, lane);
          } else {  // P_32 = L_32 X_22
            const Term t[1] = {{Lblk_t(3, 2), kLd, Xblk(2, 2), kLd}};
            gl_sum<4, 1>(t, 16 * h, 1.f, Pslot(0), kLs, lane);
          }
        }
      }
    }
    __syncthreads();
    if (*bad) break;
    if (k == kNS - 1) break;

    // ------------------------------------------------------------ B_k: L_rk = A_rk X_kk^T
    const int r0 = c0 + kS, n2 = kB - r0;
    if (warp < n2 / 16) {
      const int rg = lane >> 3, cg = lane & 7;
      const int r = r0 + 16 * warp + 4 * rg;
      const float* xt = Xdiag_t(k);
      float acc[4][4];
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[u][0] = acc[u][1] = acc[u][2] = acc[u][3] = 0.f;
#pragma unroll 2
      for (int m4 = 0; m4 < kS / 4; ++m4) {
        float4 av[4], bv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) av[u] = ld4(W + (r + u) * kLd + c0 + 4 * m4);
#pragma unroll
        for (int q = 0; q < 4; ++q) bv[q] = ld4(xt + (4 * m4 + q) * kLs + 4 * cg);
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float s = comp(av[u], q);
            acc[u][0] = fmaf(s, bv[q].x, acc[u][0]);
            acc[u][1] = fmaf(s, bv[q].y, acc[u][1]);
            acc[u][2] = fmaf(s, bv[q].z, acc[u][2]);
            acc[u][3] = fmaf(s, bv[q].w, acc[u][3]);
          }
      }
#pragma unroll
      for (int v = 0; v < 4; ++v)
        st4(Lt + (c0 + 4 * cg + v) * kLd + r, make_float4(acc[0][v], acc[1][v], acc[2][v], acc[3][v]));
    }
    __syncthreads();

    // ------------------------------------------------------------ C_k: A_rc -= L_rk L_ck^T
    // warp items: 16-row x 32-column rectangles of the trailing block that reach the lower
    // triangle; lane (rg, cg) owns a 4 x 4 tile
    {
      const int nrb = n2 / 16, ncb = n2 / 32;
      for (int item = warp; item < nrb * ncb; item += kThreads / 32) {
        const int rb = item / ncb, cb = item % ncb;
        if (32 * cb > 16 * rb + 15) continue;
        const int i = r0 + 16 * rb + 4 * (lane >> 3), j = r0 + 32 * cb + 4 * (lane & 7);
        float acc[4][4];
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[u][0] = acc[u][1] = acc[u][2] = acc[u][3] = 0.f;
        const float* lp = Lt + c0 * kLd;
#pragma unroll 8
        for (int m = 0; m < kS; ++m) {
          const float4 li = ld4(lp + m * kLd + i), lj = ld4(lp + m * kLd + j);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float s = comp(li, u);
            acc[u][0] = fmaf(s, lj.x, acc[u][0]);
            acc[u][1] = fmaf(s, lj.y, acc[u][1]);
            acc[u][2] = fmaf(s, lj.z, acc[u][2]);
            acc[u][3] = fmaf(s, lj.w, acc[u][3]);
          }
        }
        // the whole tile is written back: entries right of the diagonal are never read
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float* wp = W + (i + u) * kLd + j;
          float4 w = ld4(wp);
          w.x -= acc[u][0];
          w.y -= acc[u][1];
          w.z -= acc[u][2];
          w.w -= acc[u][3];
          st4(wp, w);
        }
      }
    }
    __syncthreads();
  }
  if (*bad) {
    if (tid == 0) atomicOr(status, kStatusNotSpd);
    return;
  }

  // ---------------------------------------------------------------- bottom block row of X
  // X_3j = -X_33 P_3j, j = 0..2: twelve 8-row pieces over the eight warps
  for (int item = warp; item < 12; item += kThreads / 32) {
    const int j = item >> 2, part = item & 3;
    const Term t[1] = {{Xdiag_t(3), kLs, Pslot(j == 0 ? 2 : j == 1 ? 4 : 0), kLs}};
    gl_sum<2, 1>(t, 8 * part, -1.f, Xblk(3, j), kLd, lane);
  }
  __syncthreads();

  // ---------------------------------------------------------------- X out (zero above the
  // diagonal sub-blocks and outside nb x nb)
  {
    const int c4 = tid & 31, i0 = tid >> 5;
#pragma unroll 4
    for (int p = 0; p < kB / 8; ++p) {
      const int i = i0 + 8 * p, j = 4 * c4;
      float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
      if ((j >> 5) <= (i >> 5)) w = ld4(W + i * kLd + j);
      if (i >= nb) w = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j + 0 >= nb) w.x = 0.f;
      if (j + 1 >= nb) w.y = 0.f;
      if (j + 2 >= nb) w.z = 0.f;
      if (j + 3 >= nb) w.w = 0.f;
      st4(Linv + i * kB + j, w);
    }
  }
}

}  // namespace

cudaError_t potrf_trtri(const float* A, long long lda, int nb, const double* shift, float* Linv, unsigned* status,
                        cudaStream_t s, int* n_launched, bool pdl) {
  cudaError_t e = cudaFuncSetAttribute(potrf_trtri_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, potrf_trtri_kernel, A, lda, nb, shift, Linv, status);
  if (e != cudaSuccess) return e;
  *n_launched += 1;
  return cudaGetLastError();
}

}  // namespace ispa
