// ispa_api.cu -- the C ABI declared in include/ispa.h: argument validation, TMA tensor maps,
// kernel dispatch, the per-device status word, host-side layer selection.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include "../../include/ispa.h"
#include "internal.h"
#include "sgemm.h"
#include "sm100.cuh"

// Sticky status word of the current device: bit (1 << ispa_status) per condition met by a kernel.
static __device__ unsigned g_ispa_status;

namespace ispa {

static std::atomic<uint64_t> g_launches{0};
static std::atomic<uint32_t> g_test_flags{0};

uint32_t test_flags() { return g_test_flags.load(); }

namespace {

constexpr int kMaxDevices = 64;
unsigned* g_status_ptr[kMaxDevices];
std::mutex g_status_mu;

// Device address of g_ispa_status on the current device (resolved once per device).
unsigned* status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_status_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_ispa_status) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<unsigned*>(p);
  }
  return g_status_ptr[dev];
}

void count(int n) { g_launches.fetch_add(static_cast<uint64_t>(n)); }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

EncodeTiledFn get_encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool make_map_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                      uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace ispa

using namespace ispa;

extern "C" {

int32_t ispa_version(void) { return 100; }

uint64_t ispa_launch_count(void) { return g_launches.load(); }

const char* ispa_status_string(ispa_status s) {
  switch (s) {
    case ISPA_OK:
      return "ok";
    case ISPA_ERR_INVALID_ARG:
      return "invalid argument";
    case ISPA_ERR_UNSUPPORTED:
      return "unsupported configuration";
    case ISPA_ERR_CUDA:
      return "CUDA runtime or launch error";
    case ISPA_ERR_NOT_SPD:
      return "G + lambda I is not positive definite (non-positive Cholesky pivot)";
    case ISPA_ERR_NONFINITE:
      return "non-finite value in an output";
    case ISPA_ERR_TIMEOUT:
      return "a bounded device wait ran out";
    case ISPA_ERR_INTERNAL:
      return "a kernel found its launch configuration unusable (internal error)";
  }
  return "unknown status";
}

ispa_status ispa_dual_stream_attn(const ispa_attn_args* a, void* stream) {
  if (!a) return ISPA_ERR_INVALID_ARG;
  if (a->dtype != ISPA_BF16 && a->dtype != ISPA_F32) return ISPA_ERR_INVALID_ARG;
  if (a->flags & ~1) return ISPA_ERR_INVALID_ARG;
  if (a->n_heads < 1 || a->head_dim < 1) return ISPA_ERR_INVALID_ARG;
  if (a->head_dim != 16 && a->head_dim != 32 && a->head_dim != 64 && a->head_dim != 128) return ISPA_ERR_UNSUPPORTED;
  const int64_t d = static_cast<int64_t>(a->n_heads) * a->head_dim;
  const int64_t lim = (1ll << 31) - 1;
  if (a->n_q < 0 || a->n_q > lim) return ISPA_ERR_INVALID_ARG;
  for (int s = 0; s < 3; ++s)
    if (a->n_kv[s] < 0 || a->n_kv[s] > lim) return ISPA_ERR_INVALID_ARG;
  if (a->n_kv[0] + a->n_kv[1] < 1) return ISPA_ERR_INVALID_ARG;
  if (!(a->softmax_scale >= 0.f) || !isfinite(a->softmax_scale)) return ISPA_ERR_INVALID_ARG;
  const size_t es = a->dtype == ISPA_BF16 ? 2 : 4;
  if (a->n_q > 0) {
    if (!a->q || !a->o_loc || !a->o_full || !a->lse_loc || !a->lse_hist) return ISPA_ERR_INVALID_ARG;
    if (a->ld_q < d || a->ld_o < d) return ISPA_ERR_INVALID_ARG;
    if (!aligned(a->q, es) || !aligned(a->o_loc, es) || !aligned(a->o_full, es) || !aligned(a->lse_loc, 4) ||
        !aligned(a->lse_hist, 4) || (a->d_out && !aligned(a->d_out, es)))
      return ISPA_ERR_INVALID_ARG;
  }
  bool biased = false;
  for (int s = 0; s < 3; ++s) {
    if (a->n_kv[s] == 0) continue;
    if (!a->k[s] || !a->v[s] || a->ld_k[s] < d || a->ld_v[s] < d) return ISPA_ERR_INVALID_ARG;
    if (!aligned(a->k[s], es) || !aligned(a->v[s], es)) return ISPA_ERR_INVALID_ARG;
    if (a->kv_bias[s]) {
      if (a->ld_bias[s] < a->n_kv[s] || !aligned(a->kv_bias[s], 4)) return ISPA_ERR_INVALID_ARG;
      biased = true;
    }
  }
  if (a->n_q == 0) return ISPA_OK;
  AttnLaunch L;
  memset(&L, 0, sizeof(L));
  L.dtype = a->dtype;
  L.n_heads = a->n_heads;
  L.head_dim = a->head_dim;
  L.n_q = a->n_q;
  L.q = a->q;
  L.ld_q = a->ld_q;
  for (int s = 0; s < 3; ++s) {
    L.n_kv[s] = a->n_kv[s];
    L.k[s] = a->k[s];
    L.v[s] = a->v[s];
    L.ld_k[s] = a->ld_k[s];
    L.ld_v[s] = a->ld_v[s];
  }
  L.scale = a->softmax_scale > 0.f ? a->softmax_scale : 1.0f / sqrtf(static_cast<float>(a->head_dim));
  L.o_loc = a->o_loc;
  L.o_full = a->o_full;
  L.d_out = a->d_out;
  L.ld_o = a->ld_o;
  L.lse_loc = a->lse_loc;
  L.lse_hist = a->lse_hist;
  L.test_flags = test_flags();
  for (int s = 0; s < 3; ++s) {
    L.bias[s] = a->n_kv[s] > 0 ? a->kv_bias[s] : nullptr;
    L.ld_bias[s] = a->ld_bias[s];
  }
  // bf16 runs on the tensor cores or not at all, unless the caller asks for the CUDA-core kernel
  const bool cuda_cores = (a->flags & ISPA_ATTN_CUDA_CORES) != 0 || a->dtype == ISPA_F32;
  if (cuda_cores && biased) return ISPA_ERR_UNSUPPORTED;  // the CUDA-core kernel takes no bias
  if (!cuda_cores && !attn_tc_supported(L)) return ISPA_ERR_UNSUPPORTED;
  L.status = status_ptr();
  if (!L.status) return ISPA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int n = 0;
  cudaError_t e = cuda_cores ? launch_attn_simt(L, st, &n) : launch_attn_tc(L, st, &n);
  count(n);
  return e == cudaSuccess ? ISPA_OK : ISPA_ERR_CUDA;
}

ispa_status ispa_accum_stats(int32_t dtype, const void* a_loc, const void* a_second, int64_t m, int32_t d, int64_t lda,
                             uint32_t flags, float* G, float* R, float* S, void* stream) {
  if (dtype != ISPA_BF16 && dtype != ISPA_F32) return ISPA_ERR_INVALID_ARG;
  if (flags & ~(ISPA_STATS_ZERO | ISPA_STATS_SECOND_IS_FULL)) return ISPA_ERR_INVALID_ARG;
  if (d < 1 || d > 65536 || m < 0 || m > (1ll << 31) - 1) return ISPA_ERR_INVALID_ARG;
  if (!G || !R || !S || !aligned(G, 4) || !aligned(R, 4) || !aligned(S, 4)) return ISPA_ERR_INVALID_ARG;
  const size_t es = dtype == ISPA_BF16 ? 2 : 4;
  if (m > 0 && (!a_loc || !a_second || lda < d || !aligned(a_loc, es) || !aligned(a_second, es)))
    return ISPA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (m == 0) {
    if (flags & ISPA_STATS_ZERO) {
      const size_t bytes = sizeof(float) * static_cast<size_t>(d) * d;
      if (cudaMemsetAsync(G, 0, bytes, st) != cudaSuccess || cudaMemsetAsync(R, 0, bytes, st) != cudaSuccess ||
          cudaMemsetAsync(S, 0, bytes, st) != cudaSuccess)
        return ISPA_ERR_CUDA;
    }
    return ISPA_OK;
  }
  StatsLaunch L;
  memset(&L, 0, sizeof(L));
  L.dtype = dtype;
  L.a_loc = a_loc;
  L.a_second = a_second;
  L.m = m;
  L.d = d;
  L.lda = lda;
  L.second_is_full = (flags & ISPA_STATS_SECOND_IS_FULL) != 0;
  L.zero = (flags & ISPA_STATS_ZERO) != 0;
  L.G = G;
  L.R = R;
  L.S = S;
  L.status = status_ptr();
  if (!L.status) return ISPA_ERR_CUDA;
  int n = 0;
  cudaError_t e = stats_tc_supported(L) ? launch_stats_tc(L, st, &n) : launch_stats_simt(L, st, &n);
  count(n);
  return e == cudaSuccess ? ISPA_OK : ISPA_ERR_CUDA;
}

ispa_status ispa_absorb_workspace_size(int32_t d, size_t* bytes) {
  if (!bytes || d < 16 || d > 16384 || d % 16) return ISPA_ERR_INVALID_ARG;
  *bytes = absorb_workspace_bytes(d, true);
  return ISPA_OK;
}

}  // extern "C"

namespace ispa {

// Shared body of ispa_absorb (parallel: five streams, larger workspace) and ispa_absorb_static
// (one stream over the library's scratch array).
int absorb_entry(const float* G, const float* R, const float* S, int32_t dtype_w, const void* W, int32_t d,
                         float lambda, uint32_t flags, float* dW, double* eps_out, void* w_new, void* ws,
                         size_t ws_bytes, void* stream, bool parallel) {
  if (d < 16 || d > 16384 || d % 16) return ISPA_ERR_INVALID_ARG;
  if (dtype_w != ISPA_BF16 && dtype_w != ISPA_F32) return ISPA_ERR_INVALID_ARG;
  if (flags & ~(ISPA_LAMBDA_REL | ISPA_W_TRANSPOSED | ISPA_WRITE_WNEW)) return ISPA_ERR_INVALID_ARG;
  if (!G || !R || !S || !W || !dW || !eps_out || !ws) return ISPA_ERR_INVALID_ARG;
  if ((flags & ISPA_WRITE_WNEW) && !w_new) return ISPA_ERR_INVALID_ARG;
  if (!(lambda >= 0.f) || !isfinite(lambda)) return ISPA_ERR_INVALID_ARG;
  const size_t es = dtype_w == ISPA_BF16 ? 2 : 4;
  if (!aligned(G, 4) || !aligned(R, 4) || !aligned(S, 4) || !aligned(dW, 4) || !aligned(eps_out, 8) ||
      !aligned(W, es) || (w_new && !aligned(w_new, es)) || !aligned(ws, 256))
    return ISPA_ERR_INVALID_ARG;
  if (ws_bytes < absorb_workspace_bytes(d, parallel)) return ISPA_ERR_INVALID_ARG;
  AbsorbLaunch L;
  memset(&L, 0, sizeof(L));
  L.G = G;
  L.R = R;
  L.S = S;
  L.dtype_w = dtype_w;
  L.W = W;
  L.d = d;
  L.lambda = lambda;
  L.lambda_rel = (flags & ISPA_LAMBDA_REL) != 0;
  L.w_transposed = (flags & ISPA_W_TRANSPOSED) != 0;
  L.write_wnew = (flags & ISPA_WRITE_WNEW) != 0;
  L.dW = dW;
  L.eps = eps_out;
  L.w_new = w_new;
  L.ws = ws;
  L.ws_bytes = ws_bytes;
  L.parallel = parallel;
  L.status = status_ptr();
  if (!L.status) return ISPA_ERR_CUDA;
  int n = 0;
  cudaError_t e = launch_absorb(L, static_cast<cudaStream_t>(stream), &n);
  count(n);
  return e == cudaSuccess ? ISPA_OK : ISPA_ERR_CUDA;
}

}  // namespace ispa

extern "C" {

ispa_status ispa_absorb(const float* G, const float* R, const float* S, int32_t dtype_w, const void* W, int32_t d,
                        float lambda, uint32_t flags, float* dW, double* eps_out, void* w_new, void* ws,
                        size_t ws_bytes, void* stream) {
  return static_cast<ispa_status>(
      absorb_entry(G, R, S, dtype_w, W, d, lambda, flags, dW, eps_out, w_new, ws, ws_bytes, stream, true));
}

ispa_status ispa_project(int32_t dtype, const void* A, int64_t m, int32_t d_in, int64_t lda, const void* W,
                         int32_t d_out, int64_t ldw, uint32_t flags, void* Y, int64_t ldy, void* stream) {
  if (dtype != ISPA_BF16 && dtype != ISPA_F32) return ISPA_ERR_INVALID_ARG;
  if (flags & ~ISPA_W_TRANSPOSED) return ISPA_ERR_INVALID_ARG;
  if (m < 0 || m > (1ll << 31) - 1 || d_in < 1 || d_out < 1) return ISPA_ERR_INVALID_ARG;
  const bool wt = (flags & ISPA_W_TRANSPOSED) != 0;
  if (lda < d_in || ldy < d_out || ldw < (wt ? d_in : d_out)) return ISPA_ERR_INVALID_ARG;
  if (m == 0) return ISPA_OK;
  if (!A || !W || !Y) return ISPA_ERR_INVALID_ARG;
  unsigned* st = status_ptr();
  if (!st) return ISPA_ERR_CUDA;
  int n = 0;
  cudaError_t e;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == ISPA_F32) {
    e = sgemm(false, wt, static_cast<int>(m), d_out, d_in, 1.f, static_cast<const float*>(A), lda,
              static_cast<const float*>(W), ldw, 0.f, static_cast<float*>(Y), ldy, false, s, &n);
  } else {
    ProjLaunch L{0, A, m, d_in, d_out, lda, W, ldw, wt, Y, ldy, st};
    if (!proj_tc_supported(L)) return ISPA_ERR_UNSUPPORTED;
    e = launch_proj_tc(L, s, &n);
  }
  count(n);
  return e == cudaSuccess ? ISPA_OK : ISPA_ERR_CUDA;
}

ispa_status ispa_quantize_e4m3(int32_t dtype, const void* X, int64_t rows, int32_t cols, int64_t ldx, uint32_t flags,
                               uint8_t* q, int64_t ldq, float* scale, void* stream) {
  if (dtype != ISPA_BF16 && dtype != ISPA_F32) return ISPA_ERR_INVALID_ARG;
  if (flags & ~ISPA_QUANT_COLUMNS) return ISPA_ERR_INVALID_ARG;
  if (rows < 0 || rows > (1ll << 31) - 1 || cols < 0) return ISPA_ERR_INVALID_ARG;
  const bool columns = (flags & ISPA_QUANT_COLUMNS) != 0;
  if (ldx < cols || ldq < (columns ? rows : cols)) return ISPA_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) return ISPA_OK;
  const size_t es = dtype == ISPA_BF16 ? 2 : 4;
  if (!X || !q || !scale || !aligned(X, es) || !aligned(scale, 4)) return ISPA_ERR_INVALID_ARG;
  if (!status_ptr()) return ISPA_ERR_CUDA;
  QuantLaunch L{dtype, X, rows, cols, ldx, columns, q, ldq, scale};
  int n = 0;
  cudaError_t e = launch_quant_e4m3(L, static_cast<cudaStream_t>(stream), &n);
  count(n);
  return e == cudaSuccess ? ISPA_OK : ISPA_ERR_CUDA;
}

ispa_status ispa_project_w8a8(const uint8_t* qa, const float* sa, int64_t m, int32_t d_in, int64_t lda, const uint8_t* qw,
                              const float* sw, int32_t d_out, int64_t ldw, void* Y, int64_t ldy, void* stream) {
  if (m < 0 || m > (1ll << 31) - 1 || d_in < 1 || d_out < 1) return ISPA_ERR_INVALID_ARG;
  if (lda < d_in || ldw < d_in || ldy < d_out) return ISPA_ERR_INVALID_ARG;
  if (m == 0) return ISPA_OK;
  if (!qa || !sa || !qw || !sw || !Y || !aligned(sa, 4) || !aligned(sw, 4) || !aligned(Y, 2)) return ISPA_ERR_INVALID_ARG;
  unsigned* st = status_ptr();
  if (!st) return ISPA_ERR_CUDA;
  W8A8Launch L{qa, sa, m, d_in, lda, qw, sw, d_out, ldw, Y, ldy, st};
  if (!w8a8_supported(L)) return ISPA_ERR_UNSUPPORTED;
  int n = 0;
  cudaError_t e = launch_w8a8(L, static_cast<cudaStream_t>(stream), &n);
  count(n);
  return e == cudaSuccess ? ISPA_OK : ISPA_ERR_CUDA;
}

ispa_status ispa_tempcache_match(int32_t n_heads, int32_t head_dim, const void* k_new, int64_t n_new, int64_t ld_new,
                                 const void* k_cache, int64_t n_cache, int64_t ld_cache, const float* inv_norm,
                                 int64_t ld_state, int32_t* idx_out, float* sim_out, void* stream) {
  if (n_heads < 1 || (head_dim != 64 && head_dim != 128)) return ISPA_ERR_UNSUPPORTED;
  const int64_t d = static_cast<int64_t>(n_heads) * head_dim;
  if (n_new < 0 || n_new > (1ll << 30) || n_cache < 0 || n_cache >= (1ll << 20)) return ISPA_ERR_INVALID_ARG;
  if (n_new == 0) return ISPA_OK;
  if (!k_new || !idx_out || !sim_out || ld_new < d || (ld_new % 8)) return ISPA_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(idx_out, 4) || !aligned(sim_out, 4)) return ISPA_ERR_INVALID_ARG;
  if (n_cache > 0 && (!k_cache || !inv_norm || ld_cache < d || (ld_cache % 8) || ld_state < n_cache ||
                      (ld_state % 4) || !aligned(k_cache, 16) || !aligned(inv_norm, 16)))
    return ISPA_ERR_INVALID_ARG;
  unsigned* st = status_ptr();
  if (!st) return ISPA_ERR_CUDA;
  TcMatchLaunch L{n_heads, head_dim, k_new, n_new, ld_new, k_cache, n_cache, ld_cache, inv_norm, ld_state,
                  idx_out, sim_out, st};
  int n = 0;
  cudaError_t e = launch_tc_match(L, static_cast<cudaStream_t>(stream), &n);
  count(n);
  return e == cudaSuccess ? ISPA_OK : ISPA_ERR_CUDA;
}

ispa_status ispa_tempcache_merge(int32_t n_heads, int32_t head_dim, void* k_cache, void* v_cache, int64_t ld_cache,
                                 int64_t capacity, int64_t n_cache, int32_t* count_, float* bias, float* inv_norm,
                                 int64_t ld_state, int32_t* n_valid, const void* k_new, const void* v_new,
                                 int64_t n_new, int64_t ld_new, const int32_t* idx, const float* sim, float threshold,
                                 void* stream) {
  if (n_heads < 1 || head_dim < 1 || head_dim > 128 || head_dim % 32) return ISPA_ERR_UNSUPPORTED;
  const int64_t d = static_cast<int64_t>(n_heads) * head_dim;
  if (n_new < 0 || n_cache < 0 || n_cache >= (1ll << 20) || capacity < n_cache + n_new) return ISPA_ERR_INVALID_ARG;
  if (isnan(threshold)) return ISPA_ERR_INVALID_ARG;
  if (n_new == 0) return ISPA_OK;
  if (!tc_merge_supported(n_new)) return ISPA_ERR_UNSUPPORTED;
  if (!k_cache || !v_cache || !count_ || !bias || !inv_norm || !n_valid || !k_new || !v_new || !idx || !sim)
    return ISPA_ERR_INVALID_ARG;
  if (ld_cache < d || ld_new < d || ld_state < capacity) return ISPA_ERR_INVALID_ARG;
  if (!aligned(k_cache, 2) || !aligned(v_cache, 2) || !aligned(k_new, 2) || !aligned(v_new, 2) ||
      !aligned(count_, 4) || !aligned(bias, 4) || !aligned(inv_norm, 4) || !aligned(n_valid, 4) ||
      !aligned(idx, 4) || !aligned(sim, 4))
    return ISPA_ERR_INVALID_ARG;
  unsigned* st = status_ptr();
  if (!st) return ISPA_ERR_CUDA;
  TcMergeLaunch L{n_heads, head_dim, k_cache, v_cache, ld_cache, n_cache, count_, bias, inv_norm, ld_state, n_valid,
                  k_new, v_new, n_new, ld_new, idx, sim, threshold, st};
  int n = 0;
  cudaError_t e = launch_tc_merge(L, static_cast<cudaStream_t>(stream), &n);
  count(n);
  return e == cudaSuccess ? ISPA_OK : ISPA_ERR_CUDA;
}

ispa_status ispa_select_layers(const double* eps, int32_t n_layers, int32_t k, int32_t* idx_out, uint8_t* mask_out) {
  if (!eps || n_layers < 0 || k < 0 || k > n_layers) return ISPA_ERR_INVALID_ARG;
  if (k > 0 && !idx_out) return ISPA_ERR_INVALID_ARG;
  std::vector<int32_t> order(static_cast<size_t>(n_layers));
  for (int32_t i = 0; i < n_layers; ++i) order[i] = i;
  // ascending eps, NaN after every number, ties to the lower layer index (stable sort on index order)
  std::stable_sort(order.begin(), order.end(), [eps](int32_t x, int32_t y) {
    const bool nx = isnan(eps[x]), ny = isnan(eps[y]);
    if (nx != ny) return ny;  // the number comes first
    if (nx) return false;
    return eps[x] < eps[y];
  });
  std::vector<int32_t> chosen(order.begin(), order.begin() + k);
  std::sort(chosen.begin(), chosen.end());
  bool nan_selected = false;
  for (int32_t i = 0; i < k; ++i) {
    idx_out[i] = chosen[i];
    if (isnan(eps[chosen[i]])) nan_selected = true;
  }
  if (mask_out) {
    for (int32_t i = 0; i < n_layers; ++i) mask_out[i] = 0;
    for (int32_t i = 0; i < k; ++i) mask_out[chosen[i]] = 1;
  }
  return nan_selected ? ISPA_ERR_NONFINITE : ISPA_OK;
}

ispa_status ispa_test_set_flags(uint32_t flags) {
  if (flags & ~ISPA_TEST_ATTN_NO_LOADS) return ISPA_ERR_INVALID_ARG;
  g_test_flags.store(flags);
  return ISPA_OK;
}

ispa_status ispa_peek_device_status_bits(uint32_t* bits_out) {
  if (!bits_out) return ISPA_ERR_INVALID_ARG;
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_ispa_status, sizeof(v)) != cudaSuccess) return ISPA_ERR_CUDA;
  *bits_out = v;
  return ISPA_OK;
}

ispa_status ispa_get_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ISPA_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_ispa_status, sizeof(v)) != cudaSuccess) return ISPA_ERR_CUDA;
  const unsigned zero = 0;
  if (cudaMemcpyToSymbol(g_ispa_status, &zero, sizeof(zero)) != cudaSuccess) return ISPA_ERR_CUDA;
  if (v & kStatusInternal) return ISPA_ERR_INTERNAL;
  if (v & kStatusTimeout) return ISPA_ERR_TIMEOUT;
  if (v & kStatusNotSpd) return ISPA_ERR_NOT_SPD;
  if (v & kStatusNonFinite) return ISPA_ERR_NONFINITE;
  return ISPA_OK;
}

}  // extern "C"
