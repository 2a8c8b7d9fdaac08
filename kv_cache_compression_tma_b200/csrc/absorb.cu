// absorb.cu -- closed-form ridge absorb and reconstruction error on one GPU.
//
// ISPA summary, section 2, stage 2 ("Layer Absorb"): the weight modulation minimising
//   ||A_loc (W + dW) - A_full W||_F^2 + lam ||dW||_F^2
// is dW = (G + lam I)^-1 R W with G = A_loc^T A_loc, R = A_loc^T (A_full - A_loc).  Section 2,
// "Dynamic Layer Selection", ranks layers by the reconstruction error eps after the absorb.
//
// Steps (all fp32 storage, fp64 where noted), workspace provided by the caller:
//   W32 = W (widened / transposed to d_in x d_out)
//   lam = lambda or lambda * trace(G) / d               (fp64 trace)
//   Lm  = G (copy; lam is added to each diagonal block by the diagonal-block kernel)
//   B   = R W32                                        (GEMM)
//   Lm  = chol(Lm) blocked by 128: diagonal block (Cholesky + explicit inverse, one CTA), panel
//         L21 = A21 L11^-T (GEMM), trailing A22 -= L21 L21^T (lower-triangle GEMM)
//   Y   = L^-1 B    blocked forward substitution with the inverted diagonal blocks (GEMMs)
//   dW  = L^-T Y    one stream: blocked back substitution (GEMMs); several streams, narrow layers:
//                   the forward substitution also carries M = L^-1 (L [Y | M] = [B | I]) and
//                   dW = M^T Y is accumulated block row by block row, dW = sum_k M_k^T Y_k, as each
//                   row becomes final, so that only one substitution step and one dW update are
//                   left after the last diagonal block; wide layers (d >= 3072): outer blocks of
//                   512, both substitutions through X_KK, the inverse of each 512-wide diagonal
//                   block (built from the 128-wide inverses), with K = 512 updates
//   P   = W32 W32^T (lower triangle; one tf32 product for a bf16 weight, whose values are tf32
//         numbers), into the factor's buffer once it is no longer needed
//   eps = <S, P> - 2 <dW, B> + ||Y||^2 - lam ||dW||^2     (deterministic fp64 reductions),
//         where <S, P> = tr(S W W^T) = <W, S W>
// The last identity is the data term of the objective expanded with G dW = L L^T dW - lam dW and
// L^T dW = Y.  eps_rel = eps / <W, S W>, the share of the missing-history signal ||D W||^2 that the
// absorb does not recover.
#include <math.h>

#include <mutex>

#include "chol.h"
#include "gemm_tc.h"
#include "internal.h"
#include "sgemm.h"
#include "sm100.cuh"

namespace ispa {
namespace {

constexpr int kPB = 128;          // panel width of the blocked factorisation
constexpr int kTwoLevelMinD = 3072;  // from this width on, the absorb runs the two-level schedule
constexpr int kRedBlocks = 512;   // fixed grid of the eps reduction (deterministic)
constexpr int kRedThreads = 256;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct WsLayout {
  size_t w32, b, lm, y, sw, linv, part, scal, total;
};

// Serial layout: W32, B, the factor (later W W^T), Y, inverted diagonal blocks, partials, scalars.
// Parallel layout: Y is the d x 2d right-hand side [Y | M] of the extended forward substitution (wide
// layers: Y, then the 512-wide inverses X_KK and a 512 x d staging block), and a separate buffer lets
// W W^T run concurrently with the factorisation.
WsLayout ws_layout(int d, bool parallel) {
  WsLayout L;
  const size_t mat = align256(sizeof(float) * static_cast<size_t>(d) * d);
  const int nb = (d + kPB - 1) / kPB;
  size_t off = 0;
  L.w32 = off;
  off += mat;
  L.b = off;
  off += mat;
  L.lm = off;
  off += mat;
  L.y = off;
  off += parallel ? 2 * mat : mat;
  if (parallel) {
    L.sw = off;
    off += mat;
  } else {
    L.sw = L.lm;
  }
  L.linv = off;
  off += align256(sizeof(float) * static_cast<size_t>(nb) * kPB * kPB);
  L.part = off;
  off += align256(sizeof(double) * 4 * kRedBlocks);
  L.scal = off;
  off += align256(sizeof(double) * 4);
  L.total = off;
  return L;
}

// Library-owned auxiliary streams and events of one device (created on first use, kept for the
// process lifetime).  sc carries the factorisation's critical path at the device's highest stream
// priority, so that its one-CTA diagonal kernels are dispatched ahead of the wide GEMMs beside it.
// The host-side enqueue of one parallel absorb holds the device's mutex.
struct AuxResources {
  cudaStream_t sc = nullptr, sa = nullptr, sb = nullptr, se = nullptr, sd = nullptr, sx = nullptr;
  static constexpr int kEvents = 2 * 128 + 16;
  cudaEvent_t ev[kEvents];
  bool ready = false;
  std::mutex mu;
};
constexpr int kMaxDevices = 64;
AuxResources g_aux[kMaxDevices];
std::mutex g_aux_init_mu;

AuxResources* aux_resources() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  AuxResources* r = &g_aux[dev];
  std::lock_guard<std::mutex> lk(g_aux_init_mu);
  if (!r->ready) {
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) return nullptr;
    if (cudaStreamCreateWithPriority(&r->sc, cudaStreamNonBlocking, greatest) != cudaSuccess) return nullptr;
    if (cudaStreamCreateWithFlags(&r->sa, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    if (cudaStreamCreateWithFlags(&r->sb, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    if (cudaStreamCreateWithFlags(&r->se, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    if (cudaStreamCreateWithFlags(&r->sd, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    if (cudaStreamCreateWithPriority(&r->sx, cudaStreamNonBlocking, greatest) != cudaSuccess) return nullptr;
    for (int i = 0; i < AuxResources::kEvents; ++i)
      if (cudaEventCreateWithFlags(&r->ev[i], cudaEventDisableTiming) != cudaSuccess) return nullptr;
    r->ready = true;
  }
  return r;
}

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

template <typename T>
__global__ void widen_w_kernel(const T* __restrict__ W, int d, int transposed, float* __restrict__ W32) {
  const long long n = static_cast<long long>(d) * d;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < n;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long i = idx / d, j = idx % d;  // W32[i][j], i = d_in, j = d_out
    W32[idx] = to_f(transposed ? W[j * d + i] : W[idx]);
  }
}

// y[i] += x[i], float4 at a time (n a multiple of 4, both 16-byte aligned)
__global__ void add_inplace_kernel(float* __restrict__ y, const float* __restrict__ x, long long n4) {
  float4* y4 = reinterpret_cast<float4*>(y);
  const float4* x4 = reinterpret_cast<const float4*>(x);
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float4 a = y4[i];
    const float4 b = x4[i];
    a.x += b.x;
    a.y += b.y;
    a.z += b.z;
    a.w += b.w;
    y4[i] = a;
  }
}

// lam = lambda (absolute) or lambda * trace(G) / d.  One block computes the trace in fp64 in a fixed
// order.  The factorisation works on a plain copy of G: the diagonal-block kernel adds lam to each
// diagonal block as it loads it (the shift only enters the diagonal, so it commutes with the
// trailing updates), and entries above the diagonal are never read.
__global__ void lambda_kernel(const float* __restrict__ G, int d, float lambda, int rel, double* scal,
                              double* eps_out) {
  __shared__ double red[256];
  double s = 0.0;
  for (int i = threadIdx.x; i < d; i += blockDim.x) s += static_cast<double>(G[static_cast<long long>(i) * d + i]);
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double lam = rel ? static_cast<double>(lambda) * red[0] / d : static_cast<double>(lambda);
    scal[0] = lam;
    scal[1] = red[0];
    eps_out[2] = lam;
  }
}

// M = I (d x d block, row stride ld)
__global__ void identity_kernel(float* __restrict__ M, long long ld, int d) {
  const long long n = static_cast<long long>(d) * d;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < n;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long i = idx / d, j = idx % d;
    M[i * ld + j] = i == j ? 1.f : 0.f;
  }
}

// partial sums: [0] <W, S W> = <S, W W^T> (P = W W^T, read on and below the diagonal, off-diagonal
// entries counted twice), [1] <dW, B>, [2] ||Y||^2, [3] ||dW||^2 (Y with row stride ldy)
__global__ void __launch_bounds__(kRedThreads) eps_partial_kernel(const float* __restrict__ S,
                                                                   const float* __restrict__ P,
                                                                   const float* __restrict__ dW,
                                                                   const float* __restrict__ B,
                                                                   const float* __restrict__ Y, int d,
                                                                   long long ldy, double* part) {
  // float4 pieces (d is a multiple of 4); the grid and the per-thread order are fixed
  __shared__ double red[4][kRedThreads];
  const int d4 = d / 4;
  const long long n4 = static_cast<long long>(d) * d4;
  double a = 0.0, b = 0.0, c = 0.0, e = 0.0;
  for (long long idx = blockIdx.x * static_cast<long long>(kRedThreads) + threadIdx.x; idx < n4;
       idx += static_cast<long long>(kRedBlocks) * kRedThreads) {
    const long long i = idx / d4;
    const int j0 = 4 * static_cast<int>(idx % d4);
    if (j0 <= i) {  // the float4 holds columns j0..j0+3 of row i: weight 2 below the diagonal, 1 on it
      const float4 sv = reinterpret_cast<const float4*>(S)[idx], pv = reinterpret_cast<const float4*>(P)[idx];
      const float s4[4] = {sv.x, sv.y, sv.z, sv.w}, p4[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const long long j = j0 + q;
        const double t = static_cast<double>(s4[q]) * p4[q];
        a += j < i ? 2.0 * t : (j == i ? t : 0.0);
      }
    }
    const float4 x = reinterpret_cast<const float4*>(dW)[idx], bb = reinterpret_cast<const float4*>(B)[idx];
    const float4 y = *reinterpret_cast<const float4*>(Y + (idx / d4) * ldy + 4 * (idx % d4));
    b += static_cast<double>(x.x) * bb.x + static_cast<double>(x.y) * bb.y + static_cast<double>(x.z) * bb.z +
         static_cast<double>(x.w) * bb.w;
    c += static_cast<double>(y.x) * y.x + static_cast<double>(y.y) * y.y + static_cast<double>(y.z) * y.z +
         static_cast<double>(y.w) * y.w;
    e += static_cast<double>(x.x) * x.x + static_cast<double>(x.y) * x.y + static_cast<double>(x.z) * x.z +
         static_cast<double>(x.w) * x.w;
  }
  red[0][threadIdx.x] = a;
  red[1][threadIdx.x] = b;
  red[2][threadIdx.x] = c;
  red[3][threadIdx.x] = e;
  __syncthreads();
  for (int w = kRedThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w)
      for (int q = 0; q < 4; ++q) red[q][threadIdx.x] += red[q][threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x < 4) part[threadIdx.x * kRedBlocks + blockIdx.x] = red[threadIdx.x][0];
}

__global__ void __launch_bounds__(kRedBlocks) eps_final_kernel(const double* part, const double* scal,
                                                                double* eps_out, unsigned* status) {
  __shared__ double red[4][kRedBlocks];
  for (int q = 0; q < 4; ++q) red[q][threadIdx.x] = part[q * kRedBlocks + threadIdx.x];
  __syncthreads();
  for (int w = kRedBlocks / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w)
      for (int q = 0; q < 4; ++q) red[q][threadIdx.x] += red[q][threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double lam = scal[0];
    const double sww = red[0][0], cross = red[1][0], yy = red[2][0], dd = red[3][0];
    const double eps = sww - 2.0 * cross + yy - lam * dd;
    eps_out[0] = eps;
    eps_out[1] = sww > 0.0 ? eps / sww : 0.0;
    eps_out[3] = sww;
    if (!isfinite(eps) || !isfinite(dd)) atomicOr(status, kStatusNonFinite);
  }
}

template <typename T>
__global__ void wnew_kernel(const T* W, const float* __restrict__ dW, int d, int transposed, T* Wn) {
  const long long n = static_cast<long long>(d) * d;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < n;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long i = idx / d, j = idx % d;  // position in W's own layout
    const float delta = transposed ? dW[j * d + i] : dW[idx];
    const float v = to_f(W[idx]) + delta;
    if constexpr (sizeof(T) == 4)
      Wn[idx] = v;
    else
      Wn[idx] = __float2bfloat16_rn(v);
  }
}

int grid_for(long long n) {
  long long b = (n + 255) / 256;
  if (b > 148 * 16) b = 148 * 16;
  if (b < 1) b = 1;
  return static_cast<int>(b);
}

#define ISPA_TRY(x)                        \
  do {                                     \
    cudaError_t e_ = (x);                  \
    if (e_ != cudaSuccess) return e_;      \
  } while (0)

}  // namespace

size_t absorb_workspace_bytes(int d, bool parallel) { return ws_layout(d, parallel).total; }

cudaError_t launch_absorb(const AbsorbLaunch& a, cudaStream_t s, int* nl) {
  const int d = a.d;
  const bool par = a.parallel;
  const WsLayout lay = ws_layout(d, par);
  uint8_t* ws = reinterpret_cast<uint8_t*>(a.ws);
  float* W32 = reinterpret_cast<float*>(ws + lay.w32);
  float* B = reinterpret_cast<float*>(ws + lay.b);
  float* Lm = reinterpret_cast<float*>(ws + lay.lm);
  float* Y = reinterpret_cast<float*>(ws + lay.y);
  float* SW = reinterpret_cast<float*>(ws + lay.sw);
  float* Linv = reinterpret_cast<float*>(ws + lay.linv);
  double* part = reinterpret_cast<double*>(ws + lay.part);
  double* scal = reinterpret_cast<double*>(ws + lay.scal);
  float* X = a.dW;
  const long long n = static_cast<long long>(d) * d;
  const int g = grid_for(n);
  const int nb = (d + kPB - 1) / kPB;

  // GEMM operands: whole matrices plus the origin of each sub-block.  Widths that are multiples of
  // 128 run the split-tf32 tensor-core GEMM; others the fp32 CUDA-core GEMM.
  struct Mat {
    const float* p;
    long long ld;
    F32Operand op;
  };
  const bool use_tc = (d % kPB) == 0;
  // wide layers are throughput-bound: two-level blocking (see below); narrow ones latency-bound
  const bool two_level = par && use_tc && d >= kTwoLevelMinD;
  Mat mR{a.R, d, {}}, mS{a.S, d, {}}, mW{W32, d, {}}, mL{Lm, d, {}}, mY{Y, d, {}}, mX{X, d, {}}, mB{B, d, {}},
      mSW{SW, d, {}}, mI{Linv, kPB, {}}, mYM{Y, 2LL * d, {}};
  if (use_tc) {
    bool ok = make_operand_maps(&mR.op, a.R, d, d, d) && make_operand_maps(&mS.op, a.S, d, d, d) &&
              make_operand_maps(&mW.op, W32, d, d, d) && make_operand_maps(&mL.op, Lm, d, d, d) &&
              make_operand_maps(&mY.op, Y, d, d, d) && make_operand_maps(&mX.op, X, d, d, d) &&
              make_operand_maps(&mB.op, B, d, d, d) && make_operand_maps(&mSW.op, SW, d, d, d) &&
              make_operand_maps(&mI.op, Linv, static_cast<uint64_t>(nb) * kPB, kPB, kPB) &&
              (!par || make_operand_maps(&mYM.op, Y, d, 2ull * d, 2ull * d));
    if (!ok) return cudaErrorInvalidValue;
  }
  // C block of matrix Cm at (cr0, cc0): C = alpha op(A) op(B) (beta == 0) or C += ... (beta == 1)
  // W32 is exact in tf32 when W is bf16: products with it skip its split (w_exact)
  const bool w_exact = a.dtype_w == 0;
  auto gemm = [&](cudaStream_t st, bool ta, bool tb, int M, int N, int K, float alpha, const Mat& A, int ar0, int ac0,
                  const Mat& Bm, int br0, int bc0, float beta, const Mat& Cm, int cr0, int cc0, bool lower,
                  bool pdl = false) -> cudaError_t {
    if (use_tc)
      return gemm_tc(ta, tb, M, N, K, alpha, A.op, ar0, ac0, Bm.op, br0, bc0, beta != 0.f, Cm.op, cr0, cc0, lower,
                     a.status, st, nl, pdl, (w_exact && &A == &mW ? 1 : 0) | (w_exact && &Bm == &mW ? 2 : 0));
    return sgemm(ta, tb, M, N, K, alpha, A.p + ar0 * A.ld + ac0, A.ld, Bm.p + br0 * Bm.ld + bc0, Bm.ld, beta,
                 const_cast<float*>(Cm.p) + cr0 * Cm.ld + cc0, Cm.ld, lower, st, nl);
  };
  // diagonal block k (+ lam on its diagonal) -> L_kk^-1; block 0 may be read straight from G
  auto diag = [&](cudaStream_t st, int k, const float* src, bool pdl = false) -> cudaError_t {
    const int r0 = k * kPB, bk = min(kPB, d - r0);
    return potrf_trtri(src + static_cast<long long>(r0) * d + r0, d, bk, scal,
                       Linv + static_cast<long long>(k) * kPB * kPB, a.status, st, nl, pdl);
  };
  // P = P L_kk^-T   (in place: one block column of width bk <= 128)
  auto panel = [&](cudaStream_t st, int k, bool pdl = false) -> cudaError_t {
    const int r0 = k * kPB, bk = min(kPB, d - r0), rem = d - r0 - bk;
    return gemm(st, false, true, rem, bk, bk, 1.f, mL, r0 + bk, r0, mI, k * kPB, 0, 0.f, mL, r0 + bk, r0, false, pdl);
  };
  // forward-substitution step k of L Y = B: Y_k = L_kk^-1 Y_k, then Y_rest -= L_rest,k Y_k
  auto fwd = [&](cudaStream_t st, int k) -> cudaError_t {
    const int r0 = k * kPB, bk = min(kPB, d - r0), rem = d - r0 - bk;
    cudaError_t e = gemm(st, false, false, bk, d, bk, 1.f, mI, k * kPB, 0, mY, r0, 0, 0.f, mY, r0, 0, false);
    if (e != cudaSuccess || rem == 0) return e;
    return gemm(st, false, false, rem, d, bk, -1.f, mL, r0 + bk, r0, mY, r0, 0, 1.f, mY, r0 + bk, 0, false);
  };

  auto widen = [&](cudaStream_t st) -> cudaError_t {
    if (a.dtype_w == 1)
      widen_w_kernel<float><<<g, 256, 0, st>>>(reinterpret_cast<const float*>(a.W), d, a.w_transposed, W32);
    else
      widen_w_kernel<__nv_bfloat16><<<g, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(a.W), d,
                                                       a.w_transposed, W32);
    ++*nl;
    return cudaGetLastError();
  };
  lambda_kernel<<<1, 256, 0, s>>>(a.G, d, a.lambda, a.lambda_rel ? 1 : 0, scal, a.eps);
  ++*nl;
  ISPA_TRY(cudaGetLastError());

  if (!par) {
    // ---------------------------------------------------------------- one stream
    ISPA_TRY(widen(s));
    ISPA_TRY(cudaMemcpyAsync(Lm, a.G, sizeof(float) * n, cudaMemcpyDeviceToDevice, s));
    ISPA_TRY(gemm(s, false, false, d, d, d, 1.f, mR, 0, 0, mW, 0, 0, 0.f, mB, 0, 0, false));  // B = R W
    for (int k = 0; k < nb; ++k) {  // blocked right-looking Cholesky of Lm = G + lam I
      const int r0 = k * kPB, bk = min(kPB, d - r0), rem = d - r0 - bk;
      ISPA_TRY(diag(s, k, Lm));
      if (rem > 0) {
        ISPA_TRY(panel(s, k));
        // trailing lower triangle: A22 -= P P^T
        ISPA_TRY(gemm(s, false, true, rem, rem, bk, -1.f, mL, r0 + bk, r0, mL, r0 + bk, r0, 1.f, mL, r0 + bk,
                      r0 + bk, true));
      }
    }
    ISPA_TRY(cudaMemcpyAsync(Y, B, sizeof(float) * n, cudaMemcpyDeviceToDevice, s));
    for (int k = 0; k < nb; ++k) ISPA_TRY(fwd(s, k));
  } else if (two_level) {
    // ---------------------------------------------------------------- wide layers: two-level blocking
    // Outer blocks of kOuter = 4 x 128 columns.  Inside an outer block the 128-wide steps run as
    // above (diagonal block + its inverse, panel, and the update of the outer block's remaining
    // columns only); the trailing matrix and the forward substitution are then updated once per
    // outer block with K = 512 products, so the large operands are streamed a quarter as often as
    // with 128-wide updates.
    // sc: the factorisation, with lookahead: after outer block K it updates only the next outer
    //     block's columns, and sd updates the rest of the trailing matrix meanwhile;
    // sa: B = R W by outer row blocks;  se: W W^T (needed only by eps, at the end);
    // sb: W32, then the forward substitution L Y = B one outer block behind the factorisation (Y
    //     starts at zero and collects the updates of the earlier blocks by add-reduction; each row
    //     block takes its B rows just before it is solved, so the substitution does not wait for all
    //     of B), then, once L is complete, the back substitution L^T dW = Y; both take one outer
    //     block at a time through X_KK, the inverse of the block's 512-wide diagonal part (one
    //     512-deep product instead of a chain of seven 128-wide ones);
    // sx (high priority, like sc: its small products must not queue behind the wide ones): X_KK of
    //     each outer block as soon as its block column is final: the four
    //     128-wide inverses of the diagonal-block kernel go on its diagonal, and the blocks below
    //     follow by growing distance from it, X_ij = -X_ii sum_{t=j..i-1} L_it X_tj.
    // X_KK and a 512 x d staging block live in the second half of the Y region of the workspace (the
    // [Y | M] right-hand side of narrow layers).
    AuxResources* ax = aux_resources();
    if (!ax) return cudaErrorUnknown;
    std::lock_guard<std::mutex> lk(ax->mu);
    int evi = 0;
    auto signal = [&](cudaStream_t from) -> cudaEvent_t {
      cudaEvent_t ev = ax->ev[evi++];
      cudaEventRecord(ev, from);
      return ev;
    };
    auto wait = [&](cudaStream_t st, cudaEvent_t ev) { return cudaStreamWaitEvent(st, ev, 0); };
    constexpr int kInner = 4, kOuter = kInner * kPB;
    const int n_outer = (nb + kInner - 1) / kInner;
    if (n_outer > 64) return cudaErrorInvalidValue;
    float* XK = Y + n;                                                   // n_outer blocks of kOuter^2
    float* Z = XK + static_cast<long long>(n_outer) * kOuter * kOuter;  // kOuter x d
    Mat mXK{XK, kOuter, {}}, mZ{Z, d, {}};
    if (!make_operand_maps(&mXK.op, XK, static_cast<uint64_t>(n_outer) * kOuter, kOuter, kOuter) ||
        !make_operand_maps(&mZ.op, Z, kOuter, d, d))
      return cudaErrorInvalidValue;
    const cudaEvent_t e_init = signal(s);
    cudaStream_t aux[6] = {ax->sc, ax->sa, ax->sb, ax->sx, ax->sd, ax->se};
    for (cudaStream_t st : aux) ISPA_TRY(wait(st, e_init));
    ISPA_TRY(cudaMemcpyAsync(Lm, a.G, sizeof(float) * n, cudaMemcpyDeviceToDevice, ax->sc));
    ISPA_TRY(widen(ax->sb));
    const cudaEvent_t e_w32 = signal(ax->sb);
    ISPA_TRY(wait(ax->sa, e_w32));
    ISPA_TRY(wait(ax->se, e_w32));
    ISPA_TRY(gemm(ax->se, false, true, d, d, d, 1.f, mW, 0, 0, mW, 0, 0, 0.f, mSW, 0, 0, true));  // W W^T
    ISPA_TRY(cudaMemsetAsync(XK, 0, sizeof(float) * n_outer * kOuter * kOuter, ax->sx));
    cudaEvent_t e_b[64], e_xk[64];
    for (int K = 0; K < n_outer; ++K) {  // B = R W, one outer row block at a time
      const int r0 = K * kOuter, rows = min(d, r0 + kOuter) - r0;
      ISPA_TRY(gemm(ax->sa, false, false, rows, d, d, 1.f, mR, r0, 0, mW, 0, 0, 0.f, mB, r0, 0, false));
      e_b[K] = signal(ax->sa);
    }
    ISPA_TRY(cudaMemsetAsync(Y, 0, sizeof(float) * n, ax->sb));
    cudaEvent_t e_rest_prev = nullptr;
    for (int K = 0; K < n_outer; ++K) {
      const int k0 = K * kInner, k1 = min(nb, k0 + kInner), ni = k1 - k0;
      const int e0 = k1 * kPB, w = ni * kPB, xr = K * kOuter;
      // factorisation of outer block K (sc)
      for (int k = k0; k < k1; ++k) {
        const int r0 = k * kPB, c1 = r0 + kPB;
        ISPA_TRY(diag(ax->sc, k, Lm, k > 0));
        if (c1 < d) {
          ISPA_TRY(panel(ax->sc, k, true));
          if (k + 1 < k1)  // the outer block's remaining columns (rows c1..d)
            ISPA_TRY(gemm(ax->sc, false, true, d - c1, (k1 - k - 1) * kPB, kPB, -1.f, mL, c1, r0, mL, c1, r0, 1.f,
                          mL, c1, c1, true));
        }
      }
      const cudaEvent_t e_col = signal(ax->sc);  // L's block column K is final
      if (e0 < d) {
        // trailing update, K = 512: the next outer block's columns on sc (after the previous block's
        // rest update, which also covers them), everything right of them on sd
        const int wn = min(d, e0 + kOuter) - e0, e2 = e0 + wn;
        if (e_rest_prev) ISPA_TRY(wait(ax->sc, e_rest_prev));
        ISPA_TRY(gemm(ax->sc, false, true, d - e0, wn, w, -1.f, mL, e0, k0 * kPB, mL, e0, k0 * kPB, 1.f, mL, e0, e0,
                      true));
        if (e2 < d) {
          ISPA_TRY(wait(ax->sd, e_col));
          ISPA_TRY(gemm(ax->sd, false, true, d - e2, d - e2, w, -1.f, mL, e2, k0 * kPB, mL, e2, k0 * kPB, 1.f, mL, e2,
                        e2, true));
          e_rest_prev = signal(ax->sd);
        } else {
          e_rest_prev = nullptr;
        }
      }
      // X_KK (sx)
      ISPA_TRY(wait(ax->sx, e_col));
      for (int i = 0; i < ni; ++i)
        ISPA_TRY(cudaMemcpy2DAsync(XK + static_cast<long long>(xr + i * kPB) * kOuter + i * kPB, sizeof(float) * kOuter,
                                   Linv + static_cast<long long>(k0 + i) * kPB * kPB, sizeof(float) * kPB,
                                   sizeof(float) * kPB, kPB, cudaMemcpyDeviceToDevice, ax->sx));
      for (int dist = 1; dist < ni; ++dist)
        for (int j = 0; j + dist < ni; ++j) {
          const int i = j + dist;
          // T = L[i, j..i-1] X[j..i-1, j] into X_ij's place, then X_ij = -X_ii T in place (M = 128)
          ISPA_TRY(gemm(ax->sx, false, false, kPB, kPB, dist * kPB, 1.f, mL, (k0 + i) * kPB, (k0 + j) * kPB, mXK,
                        xr + j * kPB, j * kPB, 0.f, mXK, xr + i * kPB, j * kPB, false));
          ISPA_TRY(gemm(ax->sx, false, false, kPB, kPB, kPB, -1.f, mXK, xr + i * kPB, i * kPB, mXK, xr + i * kPB,
                        j * kPB, 0.f, mXK, xr + i * kPB, j * kPB, false));
        }
      e_xk[K] = signal(ax->sx);
      // forward substitution of outer block K (sb): Y_K += B_K, Y_K = X_KK Y_K through the staging
      // block, then every later row, K = 512
      ISPA_TRY(wait(ax->sb, e_xk[K]));  // after L's block column K (sx waited for it)
      ISPA_TRY(wait(ax->sb, e_b[K]));
      const long long off = static_cast<long long>(k0) * kPB * d;
      {
        const long long n4 = static_cast<long long>(w) * d / 4;
        add_inplace_kernel<<<grid_for(n4), 256, 0, ax->sb>>>(Y + off, B + off, n4);
        ISPA_TRY(cudaGetLastError());
        ++*nl;
      }
      ISPA_TRY(gemm(ax->sb, false, false, w, d, w, 1.f, mXK, xr, 0, mY, k0 * kPB, 0, 0.f, mZ, 0, 0, false));
      ISPA_TRY(cudaMemcpyAsync(Y + off, Z, sizeof(float) * w * d, cudaMemcpyDeviceToDevice, ax->sb));
      if (e0 < d)
        ISPA_TRY(gemm(ax->sb, false, false, d - e0, d, w, -1.f, mL, e0, k0 * kPB, mZ, 0, 0, 1.f, mY, e0, 0, false));
    }
    // back substitution L^T dW = Y (sb; every block of L is final once sc and sd have drained):
    // X_K = X_KK^T X_K through the staging block, then every earlier row, K = 512
    ISPA_TRY(wait(ax->sb, signal(ax->sc)));
    ISPA_TRY(wait(ax->sb, signal(ax->sd)));
    ISPA_TRY(cudaMemcpyAsync(X, Y, sizeof(float) * n, cudaMemcpyDeviceToDevice, ax->sb));
    for (int K = n_outer - 1; K >= 0; --K) {
      const int k0 = K * kInner, k1 = min(nb, k0 + kInner);
      const int w = (k1 - k0) * kPB, xr = K * kOuter;
      ISPA_TRY(wait(ax->sb, e_xk[K]));
      ISPA_TRY(gemm(ax->sb, true, false, w, d, w, 1.f, mXK, xr, 0, mX, k0 * kPB, 0, 0.f, mZ, 0, 0, false));
      ISPA_TRY(cudaMemcpyAsync(X + static_cast<long long>(k0) * kPB * d, Z, sizeof(float) * w * d,
                               cudaMemcpyDeviceToDevice, ax->sb));
      if (k0 > 0)
        ISPA_TRY(gemm(ax->sb, true, false, k0 * kPB, d, w, -1.f, mL, k0 * kPB, 0, mZ, 0, 0, 1.f, mX, 0, 0, false));
    }
    for (cudaStream_t st : aux) ISPA_TRY(wait(s, signal(st)));
  } else {
    // ---------------------------------------------------------------- five streams
    // sc: diagonal blocks, panels and the next block column's update (the critical path)
    // sa: the copy G -> Lm, then the rest of each trailing update (overlaps the next diagonal
    //     block: lookahead)
    // sb: W32, B = R W, then the forward substitution of L [Y | M] = [B | I] one step behind the
    //     factorisation, each step followed by dW += M_k^T Y_k
    // se: W W^T by 256-row bands once B is done (needed only by eps), so that it never fills the
    //     SMs that the critical path needs
    AuxResources* ax = aux_resources();
    if (!ax) return cudaErrorUnknown;
    std::lock_guard<std::mutex> lk(ax->mu);
    int evi = 0;
    auto signal = [&](cudaStream_t from) -> cudaEvent_t {
      cudaEvent_t ev = ax->ev[evi++];
      cudaEventRecord(ev, from);
      return ev;
    };
    auto wait = [&](cudaStream_t st, cudaEvent_t ev) { return cudaStreamWaitEvent(st, ev, 0); };
    const long long ldym = 2LL * d;
    const cudaEvent_t e_init = signal(s);
    cudaStream_t aux[4] = {ax->sc, ax->sa, ax->sb, ax->se};
    for (cudaStream_t st : aux) ISPA_TRY(wait(st, e_init));
    // enqueued first so that its CTA is placed before the wide kernels fill the SMs
    ISPA_TRY(diag(ax->sc, 0, a.G));
    ISPA_TRY(cudaMemcpyAsync(Lm, a.G, sizeof(float) * n, cudaMemcpyDeviceToDevice, ax->sa));
    ISPA_TRY(wait(ax->sc, signal(ax->sa)));  // the copy lands before panel 0 writes into it
    ISPA_TRY(widen(ax->sb));
    // B = R W in two row halves, so that about half of the SMs stay free for the first panel
    const int half = ((nb + 1) / 2) * kPB < d ? ((nb + 1) / 2) * kPB : d;
    ISPA_TRY(gemm(ax->sb, false, false, half, d, d, 1.f, mR, 0, 0, mW, 0, 0, 0.f, mB, 0, 0, false));
    if (half < d)
      ISPA_TRY(gemm(ax->sb, false, false, d - half, d, d, 1.f, mR, half, 0, mW, 0, 0, 0.f, mB, half, 0, false));
    ISPA_TRY(wait(ax->se, signal(ax->sb)));
    for (int r0 = 0; r0 < d; r0 += 2 * kPB) {  // rows r0.. of W W^T, columns up to the band's diagonal
      const int bm = min(2 * kPB, d - r0);
      ISPA_TRY(gemm(ax->se, false, true, bm, r0 + bm, d, 1.f, mW, r0, 0, mW, 0, 0, 0.f, mSW, r0, 0, false));
    }
    ISPA_TRY(cudaMemcpy2DAsync(Y, sizeof(float) * ldym, B, sizeof(float) * d, sizeof(float) * d, d,
                               cudaMemcpyDeviceToDevice, ax->sb));
    identity_kernel<<<g, 256, 0, ax->sb>>>(Y + d, ldym, d);
    ++*nl;
    ISPA_TRY(cudaGetLastError());
    ISPA_TRY(cudaMemsetAsync(X, 0, sizeof(float) * n, ax->sb));
    cudaEvent_t e_rest_prev = nullptr;
    for (int k = 0; k < nb; ++k) {
      const int r0 = k * kPB, bk = min(kPB, d - r0), rem = d - r0 - bk;
      const int mk = min(d, (k + 1) * kPB);  // nonzero columns of row block k of M
      // the critical path's kernel -> kernel edges use programmatic dependent launch (its kernels are
      // narrow, so CTAs that start early and wait hold few SMs; the wide kernels of the other
      // streams launch normally, so that their waiting CTAs never hold the SMs the critical path
      // needs)
      if (k > 0) ISPA_TRY(diag(ax->sc, k, Lm, true));
      if (rem > 0) ISPA_TRY(panel(ax->sc, k, true));
      const cudaEvent_t e_panel = signal(ax->sc);
      ISPA_TRY(wait(ax->sb, e_panel));
      // forward step k on [Y | M] (columns past d + mk are still the identity's zeros)
      ISPA_TRY(gemm(ax->sb, false, false, bk, d + mk, bk, 1.f, mI, k * kPB, 0, mYM, r0, 0, 0.f, mYM, r0, 0, false));
      if (rem > 0)
        ISPA_TRY(gemm(ax->sb, false, false, rem, d + mk, bk, -1.f, mL, r0 + bk, r0, mYM, r0, 0, 1.f, mYM, r0 + bk, 0,
                      false));
      // dW[0:mk] += M_k^T Y_k
      ISPA_TRY(gemm(ax->sb, true, false, mk, d, bk, 1.f, mYM, r0, d, mYM, r0, 0, 1.f, mX, 0, 0, false));
      if (rem > 0) {
        const int c1 = r0 + bk, bk1 = min(kPB, rem), c2 = c1 + bk1;
        // the previous step's rest update also covers block column k+1: order the two
        if (e_rest_prev) ISPA_TRY(wait(ax->sc, e_rest_prev));
        ISPA_TRY(gemm(ax->sc, false, true, rem, bk1, bk, -1.f, mL, c1, r0, mL, c1, r0, 1.f, mL, c1, c1, true));
        if (rem > bk1) {
          ISPA_TRY(wait(ax->sa, e_panel));
          ISPA_TRY(gemm(ax->sa, false, true, rem - bk1, rem - bk1, bk, -1.f, mL, c2, r0, mL, c2, r0, 1.f, mL, c2, c2,
                        true));
          e_rest_prev = signal(ax->sa);
        } else {
          e_rest_prev = nullptr;
        }
      }
    }
    for (cudaStream_t st : aux) ISPA_TRY(wait(s, signal(st)));
  }
  if (!par) {
    // back substitution L^T dW = Y
    ISPA_TRY(cudaMemcpyAsync(X, Y, sizeof(float) * n, cudaMemcpyDeviceToDevice, s));
    for (int k = nb - 1; k >= 0; --k) {
      const int r0 = k * kPB, bk = min(kPB, d - r0);
      // X_k = L_kk^-T X_k   (in place)
      ISPA_TRY(gemm(s, true, false, bk, d, bk, 1.f, mI, k * kPB, 0, mX, r0, 0, 0.f, mX, r0, 0, false));
      if (r0 > 0)  // X[0:r0] -= L[r0:r0+bk, 0:r0]^T X_k
        ISPA_TRY(gemm(s, true, false, r0, d, bk, -1.f, mL, r0, 0, mX, r0, 0, 1.f, mX, 0, 0, false));
    }
    ISPA_TRY(gemm(s, false, true, d, d, d, 1.f, mW, 0, 0, mW, 0, 0, 0.f, mSW, 0, 0, true));  // W W^T
  }
  eps_partial_kernel<<<kRedBlocks, kRedThreads, 0, s>>>(a.S, SW, X, B, Y, d, (par && !two_level) ? 2LL * d : d,
                                                        part);
  ++*nl;
  ISPA_TRY(cudaGetLastError());
  eps_final_kernel<<<1, kRedBlocks, 0, s>>>(part, scal, a.eps, a.status);
  ++*nl;
  ISPA_TRY(cudaGetLastError());
  if (a.write_wnew) {
    if (a.dtype_w == 1)
      wnew_kernel<float><<<g, 256, 0, s>>>(reinterpret_cast<const float*>(a.W), X, d, a.w_transposed,
                                           reinterpret_cast<float*>(a.w_new));
    else
      wnew_kernel<__nv_bfloat16><<<g, 256, 0, s>>>(reinterpret_cast<const __nv_bfloat16*>(a.W), X, d,
                                                   a.w_transposed, reinterpret_cast<__nv_bfloat16*>(a.w_new));
    ++*nl;
    ISPA_TRY(cudaGetLastError());
  }
  return cudaSuccess;
}

}  // namespace ispa
