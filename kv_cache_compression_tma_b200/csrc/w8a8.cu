// w8a8.cu -- fp8 (E4M3) quantisation and the W8A8 layer output projection on tcgen05, sm_100a.
//
// ISPA summary, section 4 (results): combined with W8A8 post-training quantisation, ISPA reaches a
// 1.86x aggregate inference speed-up.  The pages fix no quantisation format; this build reads W8A8
// as fp8 E4M3 operands with one fp32 scale per activation row and one per output column of W:
//   s_i = max_k |A_ik| / 448,  qa_ik = e4m3(A_ik / s_i),   t_j = max_k |W_kj| / 448,  qw_jk = e4m3(W_kj / t_j),
//   Y_ij = s_i t_j sum_k qa_ik qw_jk,
// rounding to the nearest E4M3 value (ties to even) and saturating at +-448; an all-zero row or
// column gets scale 1.  Divisions are IEEE fp32 divisions.
//
// Quantisation kernels: per row, one warp per row with 16-byte loads for aligned bf16 rows (the
// activations), else one CTA per row (absolute maximum by a block reduction, then the scaled
// conversion); per column, a column-maximum pass and a transposing pass through 32 x 32 tiles in
// shared memory, so that the quantised weight is stored K-major ([d_out, d_in]) for the GEMM.
//
// GEMM: one CTA computes a 128 x 256 tile of Y.  Warp roles (192 threads):
//   warp 0      TMA producer: 128-byte K chunks (128 fp8) of the qa tile (one {128 B, 128 rows} box)
//               and of the qw tile (one {128 B, 256 rows} box), 128-byte swizzle, 4-stage ring;
//   warp 1      TMEM owner + single-thread MMA issuer: tcgen05.mma.kind::f8f6f4, M = 128, N = 256,
//               K = 32, fp32 accumulation in TMEM (256 columns);
//   warps 2..5  epilogue, thread = row = TMEM lane: Y = acc * s_i * t_j rounded to bf16, staged in
//               the free stage buffers (128-byte swizzle) and written by bulk tensor stores.
// Every barrier wait is bounded (see sm100.cuh); a timeout records ISPA_ERR_TIMEOUT and unwinds.
#include <cuda_fp8.h>
#include <string.h>

#include "internal.h"
#include "sm100.cuh"

namespace ispa {
namespace {

constexpr float kE4m3Max = 448.f;

__device__ __forceinline__ float load_as_float(const __nv_bfloat16* p, long long i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ float load_as_float(const float* p, long long i) { return p[i]; }

// x -> E4M3, round to nearest even, saturating finite values at +-448.
__device__ __forceinline__ uint8_t to_e4m3(float x) {
  uint16_t r;
  asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %2, %1;\n\tmov.b16 %0, t;\n\t}" : "=h"(r) : "f"(x), "f"(0.f));
  return static_cast<uint8_t>(r & 0xFF);
}

__device__ __forceinline__ float block_max_256(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x < 32) {
    float w = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) w = fmaxf(w, __shfl_xor_sync(0xffffffffu, w, o));
    if (threadIdx.x == 0) red[0] = w;
  }
  __syncthreads();
  return red[0];
}

// per-row scales; q [rows, cols] with row stride ldq bytes
template <typename T>
__global__ void __launch_bounds__(256) quant_rows_kernel(const T* __restrict__ X, long long ldx, int cols,
                                                          uint8_t* __restrict__ q, long long ldq,
                                                          float* __restrict__ scale) {
  __shared__ float red[32];
  const long long row = blockIdx.x;
  const T* x = X + row * ldx;
  float amax = 0.f;
  for (int c = threadIdx.x; c < cols; c += blockDim.x) amax = fmaxf(amax, fabsf(load_as_float(x, c)));
  amax = block_max_256(amax, red);
  const float s = amax > 0.f ? __fdiv_rn(amax, kE4m3Max) : 1.f;
  uint8_t* qr = q + row * ldq;
  for (int c = threadIdx.x; c < cols; c += blockDim.x) qr[c] = to_e4m3(__fdiv_rn(load_as_float(x, c), s));
  if (threadIdx.x == 0) scale[row] = s;
}

// per-row scales, one warp per row: bf16 rows whose length is a multiple of 8 and whose start is
// 16-byte aligned, read as 16-byte vectors (the second pass finds the row in cache); 8 codes per
// 8-byte store
__global__ void __launch_bounds__(256) quant_rows_bf16_vec_kernel(const __nv_bfloat16* __restrict__ X, long long ldx,
                                                                   long long rows, int cols, uint8_t* __restrict__ q,
                                                                   long long ldq, float* __restrict__ scale) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint4* x = reinterpret_cast<const uint4*>(X + row * ldx);
  const int nv = cols / 8;
  float amax = 0.f;
  for (int i = lane; i < nv; i += 32) {
    const uint4 w = x[i];
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k)
      amax = max3f(amax, fabsf(__uint_as_float(u[k] << 16)), fabsf(__uint_as_float(u[k] & 0xFFFF0000u)));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = amax > 0.f ? __fdiv_rn(amax, kE4m3Max) : 1.f;
  uint2* qr = reinterpret_cast<uint2*>(q + row * ldq);
  for (int i = lane; i < nv; i += 32) {
    const uint4 w = x[i];
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t lo = to_e4m3(__fdiv_rn(__uint_as_float(u[k] << 16), s));
      const uint32_t hi = to_e4m3(__fdiv_rn(__uint_as_float(u[k] & 0xFFFF0000u), s));
      packed[k >> 1] |= (lo | (hi << 8)) << (16 * (k & 1));
    }
    qr[i] = make_uint2(packed[0], packed[1]);
  }
  if (lane == 0) scale[row] = s;
}

// per-column scales of X [rows, cols]
template <typename T>
__global__ void __launch_bounds__(256) col_scale_kernel(const T* __restrict__ X, long long ldx, long long rows,
                                                         int cols, float* __restrict__ scale) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  float amax = 0.f;
  for (long long r = 0; r < rows; ++r) amax = fmaxf(amax, fabsf(load_as_float(X, r * ldx + c)));
  scale[c] = amax > 0.f ? __fdiv_rn(amax, kE4m3Max) : 1.f;
}

// qt[c, r] = e4m3(X[r, c] / scale[c]) through 32 x 32 shared-memory tiles (qt row stride ldq bytes)
template <typename T>
__global__ void __launch_bounds__(256) quant_cols_t_kernel(const T* __restrict__ X, long long ldx, long long rows,
                                                            int cols, const float* __restrict__ scale,
                                                            uint8_t* __restrict__ qt, long long ldq) {
  __shared__ uint8_t tile[32][33];
  const long long r0 = static_cast<long long>(blockIdx.y) * 32;
  const int c0 = blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 8 rows of 32 threads
  for (int i = ty; i < 32; i += 8) {
    const long long r = r0 + i;
    const int c = c0 + tx;
    uint8_t v = 0;
    if (r < rows && c < cols) v = to_e4m3(__fdiv_rn(load_as_float(X, r * ldx + c), scale[c]));
    tile[i][tx] = v;
  }
  __syncthreads();
  for (int i = ty; i < 32; i += 8) {
    const int c = c0 + i;
    const long long r = r0 + tx;
    if (c < cols && r < rows) qt[static_cast<long long>(c) * ldq + r] = tile[tx][i];
  }
}

// ------------------------------------------------------------------------------------------ GEMM
constexpr int kTM = 128, kTN = 256;
constexpr int kBK = 128;                    // fp8 elements (bytes) of K per stage
constexpr int kStages = 4;
constexpr int kATileBytes = kTM * kBK;      // 16 KB
constexpr int kBTileBytes = kTN * kBK;      // 32 KB
constexpr int kStageBytes = kATileBytes + kBTileBytes;
constexpr int kThreads = 192;
constexpr int kOffBar = kStages * kStageBytes;
constexpr int kOffMisc = kOffBar + (2 * kStages + 1) * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;
static_assert(kStages * kStageBytes >= (kTN / 64) * kTM * 128, "the output tile is staged in the ring");
static_assert(kSmemBytes <= 232448, "shared memory budget");

// Instruction descriptor of tcgen05.mma.kind::f8f6f4 with E4M3 A and B (format code 0), K-major
// operands and fp32 accumulation: bits [4,6) D format (1 = f32), [7,10) A format, [10,13) B
// format, [17,23) N >> 3, [24,29) M >> 4.
constexpr uint32_t kIdescE4m3 = (1u << 4) | (static_cast<uint32_t>(kTN >> 3) << 17) |
                                (static_cast<uint32_t>(kTM >> 4) << 24);

__device__ __forceinline__ void umma_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

struct W8Params {
  int m, d_in, d_out;
  long long ldy;
  const float* sa;
  const float* sw;
  __nv_bfloat16* y;
  unsigned* status;
};

__global__ void __launch_bounds__(kThreads, 1)
    w8a8_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapW,
                   const __grid_constant__ CUtensorMap mapY, const W8Params p) {
  const int n0 = blockIdx.x * kTN, m0 = blockIdx.y * kTM;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  volatile int* never = reinterpret_cast<volatile int*>(smem + kOffMisc + 8);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_steps = p.d_in / kBK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    *never = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int k = 0; k < n_steps; ++k) {
        const int s = k % kStages;
        if (k >= kStages && !mbar_wait(empty + s, ((k / kStages) - 1) & 1, abort_flag)) {
          atomicOr(p.status, kStatusTimeout);
          *abort_flag = 1;
          break;
        }
        uint8_t* st = smem + s * kStageBytes;
        mbar_arrive_expect_tx(full + s, kStageBytes);
        tma_load_2d(st, &mapA, full + s, k * kBK, m0);  // rows past m read as zeros
        tma_load_2d(st + kATileBytes, &mapW, full + s, k * kBK, n0);
        issued = k + 1;
      }
      if (*abort_flag) {
        for (int k = issued - 1; k >= 0 && k >= issued - kStages; --k)
          mbar_wait(full + (k % kStages), (k / kStages) & 1, never);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = true;
      for (int k = 0; k < n_steps; ++k) {
        const int s = k % kStages;
        if (!mbar_wait(full + s, (k / kStages) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_u32(smem + s * kStageBytes);
        const uint32_t w_base = a_base + kATileBytes;
#pragma unroll
        for (int kk = 0; kk < kBK / 32; ++kk)  // 32 fp8 = 32 bytes along the swizzled 128-byte row
          umma_f8(tmem, sw128_desc(a_base + kk * 32, 16, 1024), sw128_desc(w_base + kk * 32, 16, 1024), kIdescE4m3,
                  (k > 0 || kk > 0) ? 1u : 0u);
        umma_commit(empty + s);
      }
      if (!ok) {
        atomicOr(p.status, kStatusTimeout);
        *abort_flag = 1;
      }
      umma_commit(acc_full);
    }
  } else {
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const bool ok = mbar_wait_warp(acc_full, 0, abort_flag);
    if (ok) {
      // Y = acc * s_i * t_j -> bf16, staged in the stage buffers (free: every load and MMA is done)
      // as four 128-byte-swizzled {64 cols, 128 rows} boxes; rows past m are clipped by the store
      tc_fence_after();
      const uint32_t addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
      const int grow = m0 + row;
      const float sa = grow < p.m ? p.sa[grow] : 0.f;
#pragma unroll 1
      for (int c = 0; c < kTN; c += 32) {
        uint32_t v[32];
        tmem_ld32(addr + c, v);
        tmem_wait_ld();
        const float4* sw4 = reinterpret_cast<const float4*>(p.sw + n0 + c);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 t0 = __ldg(sw4 + 2 * i), t1 = __ldg(sw4 + 2 * i + 1);
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(v[8 * i + 0]) * sa * t0.x, __uint_as_float(v[8 * i + 1]) * sa * t0.y);
          w.y = pack_bf16x2(__uint_as_float(v[8 * i + 2]) * sa * t0.z, __uint_as_float(v[8 * i + 3]) * sa * t0.w);
          w.z = pack_bf16x2(__uint_as_float(v[8 * i + 4]) * sa * t1.x, __uint_as_float(v[8 * i + 5]) * sa * t1.y);
          w.w = pack_bf16x2(__uint_as_float(v[8 * i + 6]) * sa * t1.z, __uint_as_float(v[8 * i + 7]) * sa * t1.w);
          const int col = c + 8 * i, q = (col & 63) >> 3;
          *reinterpret_cast<uint4*>(smem + (col >> 6) * (kTM * 128) + row * 128 + ((q ^ (row & 7)) << 4)) = w;
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    } else {
      atomicOr(p.status, kStatusTimeout);
      *abort_flag = 1;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");  // the four epilogue warps
    if (warp == 2 && lane == 0 && !*abort_flag) {
      for (int b = 0; b < kTN / 64; ++b)
        asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                         reinterpret_cast<uint64_t>(&mapY)),
                     "r"(smem_u32(smem + b * (kTM * 128))), "r"(n0 + 64 * b), "r"(m0)
                     : "memory");
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTN);
  }
}

bool make_map_u8_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t ld_bytes,
                    uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_quant_e4m3(const QuantLaunch& a, cudaStream_t s, int* n_launched) {
  if (a.rows == 0 || a.cols == 0) return cudaSuccess;
  if (!a.columns) {
    const bool vec = a.dtype == 0 && a.cols % 8 == 0 && a.ldx % 8 == 0 && a.ldq % 8 == 0 &&
                     (reinterpret_cast<uintptr_t>(a.X) & 15) == 0 && (reinterpret_cast<uintptr_t>(a.q) & 7) == 0;
    if (vec) {
      quant_rows_bf16_vec_kernel<<<static_cast<unsigned>((a.rows + 7) / 8), 256, 0, s>>>(
          static_cast<const __nv_bfloat16*>(a.X), a.ldx, a.rows, a.cols, a.q, a.ldq, a.scale);
      *n_launched += 1;
      return cudaGetLastError();
    }
    const dim3 grid(static_cast<unsigned>(a.rows));
    if (a.dtype == 0)
      quant_rows_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(a.X), a.ldx, a.cols, a.q, a.ldq,
                                             a.scale);
    else
      quant_rows_kernel<<<grid, 256, 0, s>>>(static_cast<const float*>(a.X), a.ldx, a.cols, a.q, a.ldq, a.scale);
    *n_launched += 1;
    return cudaGetLastError();
  }
  const dim3 g1((a.cols + 255) / 256);
  const dim3 g2((a.cols + 31) / 32, static_cast<unsigned>((a.rows + 31) / 32));
  if (a.dtype == 0) {
    const __nv_bfloat16* X = static_cast<const __nv_bfloat16*>(a.X);
    col_scale_kernel<<<g1, 256, 0, s>>>(X, a.ldx, a.rows, a.cols, a.scale);
    quant_cols_t_kernel<<<g2, 256, 0, s>>>(X, a.ldx, a.rows, a.cols, a.scale, a.q, a.ldq);
  } else {
    const float* X = static_cast<const float*>(a.X);
    col_scale_kernel<<<g1, 256, 0, s>>>(X, a.ldx, a.rows, a.cols, a.scale);
    quant_cols_t_kernel<<<g2, 256, 0, s>>>(X, a.ldx, a.rows, a.cols, a.scale, a.q, a.ldq);
  }
  *n_launched += 2;
  return cudaGetLastError();
}

bool w8a8_supported(const W8A8Launch& a) {
  auto al16 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; };
  return a.d_in % kBK == 0 && a.d_out % kTN == 0 && a.lda % 16 == 0 && a.ldw % 16 == 0 && a.ldy % 8 == 0 &&
         al16(a.qa) && al16(a.qw) && al16(a.Y) && al16(a.sw) && a.m <= (1ll << 30);
}

cudaError_t launch_w8a8(const W8A8Launch& a, cudaStream_t s, int* n_launched) {
  if (a.m == 0) return cudaSuccess;
  CUtensorMap mapA, mapW, mapY;
  memset(&mapA, 0, sizeof(mapA));
  memset(&mapW, 0, sizeof(mapW));
  memset(&mapY, 0, sizeof(mapY));
  if (!make_map_bf16_2d(&mapY, a.Y, a.m, a.d_out, a.ldy, 64, kTM)) return cudaErrorInvalidValue;
  if (!make_map_u8_2d(&mapA, a.qa, a.m, a.d_in, a.lda, kBK, kTM)) return cudaErrorInvalidValue;
  if (!make_map_u8_2d(&mapW, a.qw, a.d_out, a.d_in, a.ldw, kBK, kTN)) return cudaErrorInvalidValue;
  W8Params p;
  p.m = static_cast<int>(a.m);
  p.d_in = a.d_in;
  p.d_out = a.d_out;
  p.ldy = a.ldy;
  p.sa = a.sa;
  p.sw = a.sw;
  p.y = reinterpret_cast<__nv_bfloat16*>(a.Y);
  p.status = a.status;
  cudaError_t e = cudaFuncSetAttribute(w8a8_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(a.d_out / kTN, static_cast<unsigned>((a.m + kTM - 1) / kTM));
  w8a8_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(mapA, mapW, mapY, p);
  *n_launched += 1;
  return cudaGetLastError();
}

}  // namespace ispa
