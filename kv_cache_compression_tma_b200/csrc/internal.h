// internal.h -- launcher interfaces shared between the C ABI (ispa_api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ispa {

// ------------------------------------------------------------------ dual-stream attention
struct AttnLaunch {
  int dtype;  // 0 bf16, 1 f32
  int n_heads, head_dim;
  int64_t n_q;
  int64_t n_kv[3];
  const void* q;
  int64_t ld_q;
  const void* k[3];
  const void* v[3];
  int64_t ld_k[3], ld_v[3];
  float scale;
  void* o_loc;
  void* o_full;
  void* d_out;
  int64_t ld_o;
  float* lse_loc;
  float* lse_hist;
  unsigned* status;
  uint32_t test_flags;  // ISPA_TEST_* hooks (0 in normal use)
  const float* bias[3];  // optional per-key logit bias per segment, [n_heads, n_kv[s]], natural log
  int64_t ld_bias[3];
};

// Process-wide test hooks set by ispa_test_set_flags (0 = off).
uint32_t test_flags();

// tcgen05 kernel (bf16, head_dim 64/128, TMA-compatible strides); returns cudaError_t
cudaError_t launch_attn_tc(const AttnLaunch& a, cudaStream_t s, int* n_launched);
bool attn_tc_supported(const AttnLaunch& a);
// CUDA-core kernel (any supported dtype / head_dim)
cudaError_t launch_attn_simt(const AttnLaunch& a, cudaStream_t s, int* n_launched);

// ------------------------------------------------------------------ Gram statistics
struct StatsLaunch {
  int dtype;
  const void* a_loc;
  const void* a_second;
  int64_t m;
  int d;
  int64_t lda;
  bool second_is_full;
  bool zero;
  float* G;
  float* R;
  float* S;
  unsigned* status;
};
bool stats_tc_supported(const StatsLaunch& a);
cudaError_t launch_stats_tc(const StatsLaunch& a, cudaStream_t s, int* n_launched);
cudaError_t launch_stats_simt(const StatsLaunch& a, cudaStream_t s, int* n_launched);

// ------------------------------------------------------------------ absorb
struct AbsorbLaunch {
  const float* G;
  const float* R;
  const float* S;
  int dtype_w;
  const void* W;
  int d;
  float lambda;
  bool lambda_rel;
  bool w_transposed;
  bool write_wnew;
  float* dW;
  double* eps;
  void* w_new;
  void* ws;
  size_t ws_bytes;
  bool parallel;  // five streams with lookahead (larger workspace) vs one stream
  unsigned* status;
};
size_t absorb_workspace_bytes(int d, bool parallel);
cudaError_t launch_absorb(const AbsorbLaunch& a, cudaStream_t s, int* n_launched);
// argument checks + launch of the absorb (ispa_absorb: parallel; ispa_absorb_static: one stream)
int absorb_entry(const float* G, const float* R, const float* S, int32_t dtype_w, const void* W, int32_t d,
                 float lambda, uint32_t flags, float* dW, double* eps_out, void* w_new, void* ws, size_t ws_bytes,
                 void* stream, bool parallel);

// ------------------------------------------------------------------ output projection
struct ProjLaunch {
  int dtype;  // 0 bf16 (tensor cores), 1 f32
  const void* A;
  int64_t m;
  int d_in, d_out;
  int64_t lda;
  const void* W;
  int64_t ldw;
  bool w_transposed;  // W stored d_out x d_in
  void* Y;
  int64_t ldy;
  unsigned* status;
};
bool proj_tc_supported(const ProjLaunch& a);
cudaError_t launch_proj_tc(const ProjLaunch& a, cudaStream_t s, int* n_launched);

// ------------------------------------------------------------------ W8A8 (fp8 E4M3) projection
struct QuantLaunch {
  int dtype;  // 0 bf16, 1 f32
  const void* X;
  int64_t rows;
  int cols;
  int64_t ldx;
  bool columns;  // per-column scales, output transposed [cols, rows]
  uint8_t* q;
  int64_t ldq;   // bytes
  float* scale;
};
cudaError_t launch_quant_e4m3(const QuantLaunch& a, cudaStream_t s, int* n_launched);

struct W8A8Launch {
  const uint8_t* qa;
  const float* sa;
  int64_t m;
  int d_in;
  int64_t lda;  // bytes
  const uint8_t* qw;  // [d_out, d_in], K-major
  const float* sw;
  int d_out;
  int64_t ldw;  // bytes
  void* Y;      // bf16 [m, d_out]
  int64_t ldy;  // elements
  unsigned* status;
};
bool w8a8_supported(const W8A8Launch& a);
cudaError_t launch_w8a8(const W8A8Launch& a, cudaStream_t s, int* n_launched);

// ------------------------------------------------------------------ TempCache (FAST-AR)
struct TcMatchLaunch {
  int n_heads, head_dim;
  const void* k_new;
  int64_t n_new, ld_new;
  const void* k_cache;
  int64_t n_cache, ld_cache;
  const float* inv_norm;
  int64_t ld_state;
  int* idx;
  float* sim;
  unsigned* status;
};
cudaError_t launch_tc_match(const TcMatchLaunch& a, cudaStream_t s, int* n_launched);

struct TcMergeLaunch {
  int n_heads, head_dim;
  void* k_cache;
  void* v_cache;
  int64_t ld_cache, n_cache;
  int* count;
  float* bias;
  float* inv_norm;
  int64_t ld_state;
  int* n_valid;
  const void* k_new;
  const void* v_new;
  int64_t n_new, ld_new;
  const int* idx;
  const float* sim;
  float threshold;
  unsigned* status;
};
bool tc_merge_supported(int64_t n_new);
cudaError_t launch_tc_merge(const TcMergeLaunch& a, cudaStream_t s, int* n_launched);

// driver entry point for cuTensorMapEncodeTiled (resolved once through the runtime)
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn get_encode_tiled();

// 2-D bf16 row-major tensor map: `rows` x `cols` elements, row stride `ld` elements, box
// {box_cols, box_rows}, 128-byte swizzle.  Returns false if the driver rejects it.
bool make_map_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                      uint32_t box_cols, uint32_t box_rows);

}  // namespace ispa
