// attn_simt.cu -- decomposable (dual-stream) attention on CUDA cores (fp32 arithmetic).
//
// Same computation as the tensor-core kernel (ISPA summary, section 2, stage 1): one pass over
// sink, local and history keys with a separate online-softmax state (max, sum, accumulator) per
// branch and a post-hoc log-sum-exp merge.  Used for fp32 inputs and for head dims / alignments the
// tensor-core kernel does not take.  One warp handles one (query row, head); lane e holds elements
// e, e+32, ... of the head, so q.k is a warp-shuffle reduction and key rows are read coalesced.
#include <math.h>

#include "internal.h"
#include "sm100.cuh"

namespace ispa {
namespace {

constexpr int kWarpsPerBlock = 4;

template <typename T>
__device__ __forceinline__ float ld_elem(const T* p);
template <>
__device__ __forceinline__ float ld_elem<float>(const float* p) {
  return *p;
}
template <>
__device__ __forceinline__ float ld_elem<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <typename T>
__device__ __forceinline__ void st_elem(T* p, float v);
template <>
__device__ __forceinline__ void st_elem<float>(float* p, float v) {
  *p = v;
}
template <>
__device__ __forceinline__ void st_elem<__nv_bfloat16>(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}

struct SimtParams {
  int n_heads, head_dim;
  long long n_q;
  long long n_kv[3];
  const void* q;
  long long ld_q;
  const void* k[3];
  const void* v[3];
  long long ld_k[3], ld_v[3];
  float scale;
  void* o_loc;
  void* o_full;
  void* d_out;
  long long ld_o;
  float* lse_loc;
  float* lse_hist;
};

template <typename T, int EPL>
__global__ void __launch_bounds__(kWarpsPerBlock * 32) attn_simt_kernel(const SimtParams p) {
  const int lane = threadIdx.x & 31;
  const long long gw = static_cast<long long>(blockIdx.x) * kWarpsPerBlock + (threadIdx.x >> 5);
  if (gw >= p.n_q * p.n_heads) return;
  const long long row = gw / p.n_heads;
  const int head = static_cast<int>(gw % p.n_heads);
  const int hd = p.head_dim;
  const int col0 = head * hd;

  float q[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    q[i] = e < hd ? ld_elem(reinterpret_cast<const T*>(p.q) + row * p.ld_q + col0 + e) * p.scale : 0.f;
  }
  float m_b[2] = {-INFINITY, -INFINITY}, l_b[2] = {0.f, 0.f};
  float acc[2][EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) acc[0][i] = acc[1][i] = 0.f;

  for (int seg = 0; seg < 3; ++seg) {
    const int br = seg == 2 ? 1 : 0;
    const T* K = reinterpret_cast<const T*>(p.k[seg]);
    const T* V = reinterpret_cast<const T*>(p.v[seg]);
    for (long long j = 0; j < p.n_kv[seg]; ++j) {
      float part = 0.f;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        if (e < hd) part = fmaf(q[i], ld_elem(K + j * p.ld_k[seg] + col0 + e), part);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      const float m_new = fmaxf(m_b[br], part);
      const float alpha = expf(m_b[br] - m_new);  // exp(-inf) = 0 on the first key
      const float pj = expf(part - m_new);
      l_b[br] = l_b[br] * alpha + pj;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        const float vv = e < hd ? ld_elem(V + j * p.ld_v[seg] + col0 + e) : 0.f;
        acc[br][i] = fmaf(acc[br][i], alpha, pj * vv);
      }
      m_b[br] = m_new;
    }
  }
  const bool has_hist = p.n_kv[2] > 0;
  const float lse_l = m_b[0] + logf(l_b[0]);
  const float lse_h = has_hist ? m_b[1] + logf(l_b[1]) : -INFINITY;
  float w_l = 1.f, w_h = 0.f;
  if (has_hist) {
    const float mm = fmaxf(lse_l, lse_h);
    const float a = expf(lse_l - mm), b = expf(lse_h - mm);
    w_l = a / (a + b);
    w_h = b / (a + b);
  }
  T* ol = reinterpret_cast<T*>(p.o_loc) + row * p.ld_o + col0;
  T* of = reinterpret_cast<T*>(p.o_full) + row * p.ld_o + col0;
  T* od = p.d_out ? reinterpret_cast<T*>(p.d_out) + row * p.ld_o + col0 : nullptr;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    if (e >= hd) continue;
    const float vl = acc[0][i] / l_b[0];
    const float vf = has_hist ? fmaf(w_l, vl, w_h * (acc[1][i] / l_b[1])) : vl;
    st_elem(ol + e, vl);
    st_elem(of + e, vf);
    if (od) st_elem(od + e, vf - vl);
  }
  if (lane == 0) {
    p.lse_loc[static_cast<long long>(head) * p.n_q + row] = lse_l;
    p.lse_hist[static_cast<long long>(head) * p.n_q + row] = lse_h;
  }
}

template <typename T>
cudaError_t launch_t(const SimtParams& p, cudaStream_t s, int* n) {
  const long long warps = p.n_q * p.n_heads;
  const unsigned blocks = static_cast<unsigned>((warps + kWarpsPerBlock - 1) / kWarpsPerBlock);
  const int epl = (p.head_dim + 31) / 32;
  if (epl <= 1)
    attn_simt_kernel<T, 1><<<blocks, kWarpsPerBlock * 32, 0, s>>>(p);
  else if (epl == 2)
    attn_simt_kernel<T, 2><<<blocks, kWarpsPerBlock * 32, 0, s>>>(p);
  else
    attn_simt_kernel<T, 4><<<blocks, kWarpsPerBlock * 32, 0, s>>>(p);
  *n += 1;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_simt(const AttnLaunch& a, cudaStream_t s, int* n_launched) {
  if (a.n_q == 0) return cudaSuccess;
  SimtParams p;
  p.n_heads = a.n_heads;
  p.head_dim = a.head_dim;
  p.n_q = a.n_q;
  p.q = a.q;
  p.ld_q = a.ld_q;
  for (int i = 0; i < 3; ++i) {
    p.n_kv[i] = a.n_kv[i];
    p.k[i] = a.k[i];
    p.v[i] = a.v[i];
    p.ld_k[i] = a.ld_k[i];
    p.ld_v[i] = a.ld_v[i];
  }
  p.scale = a.scale;
  p.o_loc = a.o_loc;
  p.o_full = a.o_full;
  p.d_out = a.d_out;
  p.ld_o = a.ld_o;
  p.lse_loc = a.lse_loc;
  p.lse_hist = a.lse_hist;
  if (a.dtype == 1) return launch_t<float>(p, s, n_launched);
  return launch_t<__nv_bfloat16>(p, s, n_launched);
}

}  // namespace ispa
