// proj_tc.cu -- layer output projection Y = A W on tcgen05 tensor cores (bf16, sm_100a).
//
// ISPA summary, section 2, stage 3 (memory-efficient inference): after T_warm an L-Layer attends
// over its local context only and projects that output with W_new = W + dW, while an F-Layer keeps
// full attention and W.  This kernel is the projection of both: Y[m, d_out] = A[m, d_in] op(W) with
// bf16 operands, fp32 accumulation in TMEM and Y rounded to bf16 once.
//
// One CTA computes one 128 x 128 tile of Y.  Warp roles (192 threads):
//   warp 0      TMA producer: 64-wide K chunks of the A tile (K-major, one {64, 128} box) and of W
//               (W stored d_in x d_out is MN-major: two {64 N, 64 K} boxes; W stored d_out x d_in,
//               the torch Linear layout, is K-major: one {64 K, 128 N} box), 128-byte swizzle, a
//               4-stage ring, each CTA loading its own tiles
//   warp 1      TMEM owner + single-thread MMA issuer: four kind::f16 MMAs (K = 16) per chunk
//   warps 2..5  epilogue, thread = row = TMEM lane: fp32 accumulator -> bf16 -> the tile staged in
//               the free stage buffers (128-byte swizzle) -> bulk tensor stores
// Every barrier wait is bounded (see sm100.cuh); a timeout records ISPA_ERR_TIMEOUT and unwinds.
#include <string.h>

#include "internal.h"
#include "sm100.cuh"

namespace ispa {
namespace {

constexpr int kT = 128;                     // tile M = N
constexpr int kBK = 64;                     // K per stage (one 128-byte swizzle row of bf16)
constexpr int kStages = 4;
constexpr int kTileBytes = kT * kBK * 2;    // 16 KB
constexpr int kStageBytes = 2 * kTileBytes; // A, W
constexpr int kThreads = 192;
constexpr int kOffBar = kStages * kStageBytes;
constexpr int kOffMisc = kOffBar + (2 * kStages + 1) * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + slack to align the base to 1024 bytes

struct ProjParams {
  int m, d_in, d_out;
  long long ldy;
  __nv_bfloat16* y;
  unsigned* status;
};

template <bool W_KMAJOR>
__global__ void __launch_bounds__(kThreads, 1)
    proj_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapW,
                   const __grid_constant__ CUtensorMap mapY, const ProjParams p) {
  const int n0 = blockIdx.x * kT, m0 = blockIdx.y * kT;
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
    tmem_alloc(tmem_slot, kT);
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
        const int k0 = k * kBK;
        mbar_arrive_expect_tx(full + s, kStageBytes);
        tma_load_2d(st, &mapA, full + s, k0, m0);  // rows past m read as zeros
        if (W_KMAJOR) {
          tma_load_2d(st + kTileBytes, &mapW, full + s, k0, n0);
        } else {
          tma_load_2d(st + kTileBytes, &mapW, full + s, n0, k0);
          tma_load_2d(st + kTileBytes + kTileBytes / 2, &mapW, full + s, n0 + 64, k0);
        }
        issued = k + 1;
      }
      // never leave the CTA with bulk copies in flight
      if (*abort_flag) {
        for (int k = issued - 1; k >= 0 && k >= issued - kStages; --k)
          mbar_wait(full + (k % kStages), (k / kStages) & 1, never);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = true;
      constexpr uint32_t idesc = idesc_bf16_f32(kT, kT, false, !W_KMAJOR);
      for (int k = 0; k < n_steps; ++k) {
        const int s = k % kStages;
        if (!mbar_wait(full + s, (k / kStages) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_u32(smem + s * kStageBytes);
        const uint32_t w_base = a_base + kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          // K-major: 16 bf16 = 32 bytes along the swizzled row; MN-major: 16 K rows = 2048 bytes,
          // the two 64-wide N chunks 8 KB apart
          const uint64_t adesc = sw128_desc(a_base + kk * 32, 16, 1024);
          const uint64_t wdesc = W_KMAJOR ? sw128_desc(w_base + kk * 32, 16, 1024)
                                          : sw128_desc(w_base + kk * 16 * 128, kTileBytes / 2, 1024);
          umma_ss(tmem, adesc, wdesc, idesc, (k > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(empty + s);
      }
      if (!ok) {
        atomicOr(p.status, kStatusTimeout);
        *abort_flag = 1;
      }
      umma_commit(acc_full);
    }
  } else {
    // epilogue: thread = row = TMEM lane of this warp's quarter
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const bool ok = mbar_wait_warp(acc_full, 0, abort_flag);
    if (ok) {
      // the tile goes through the stage buffers (free: every load and MMA is done) as two
      // 128-byte-swizzled {64 cols, 128 rows} boxes; rows past m are clipped by the store
      tc_fence_after();
      const uint32_t addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < kT; c += 32) {
        uint32_t v[32];
        tmem_ld32(addr + c, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(v[8 * i + 0]), __uint_as_float(v[8 * i + 1]));
          w.y = pack_bf16x2(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3]));
          w.z = pack_bf16x2(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5]));
          w.w = pack_bf16x2(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7]));
          const int col = c + 8 * i, q = (col & 63) >> 3;
          *reinterpret_cast<uint4*>(smem + (col >> 6) * (kT * 128) + row * 128 + ((q ^ (row & 7)) << 4)) = w;
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    } else {
      atomicOr(p.status, kStatusTimeout);
      *abort_flag = 1;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");  // the four epilogue warps
    if (warp == 2 && lane == 0 && !*abort_flag) {
      for (int b = 0; b < kT / 64; ++b)
        asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                         reinterpret_cast<uint64_t>(&mapY)),
                     "r"(smem_u32(smem + b * (kT * 128))), "r"(n0 + 64 * b), "r"(m0)
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
    tmem_dealloc(tmem, kT);
  }
}

}  // namespace

bool proj_tc_supported(const ProjLaunch& a) {
  auto al16 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; };
  return a.dtype == 0 && a.d_in % kBK == 0 && a.d_out % kT == 0 && a.lda % 8 == 0 && a.ldw % 8 == 0 &&
         a.ldy % 8 == 0 && al16(a.A) && al16(a.W) && al16(a.Y) && a.m <= (1ll << 30);
}

cudaError_t launch_proj_tc(const ProjLaunch& a, cudaStream_t s, int* n_launched) {
  if (a.m == 0) return cudaSuccess;
  CUtensorMap mapA, mapW, mapY;
  memset(&mapA, 0, sizeof(mapA));
  memset(&mapW, 0, sizeof(mapW));
  memset(&mapY, 0, sizeof(mapY));
  if (!make_map_bf16_2d(&mapY, a.Y, a.m, a.d_out, a.ldy, 64, kT)) return cudaErrorInvalidValue;
  if (!make_map_bf16_2d(&mapA, a.A, a.m, a.d_in, a.lda, kBK, kT)) return cudaErrorInvalidValue;
  const bool wk = a.w_transposed;
  if (wk) {  // W stored d_out x d_in: rows = N, columns = K
    if (!make_map_bf16_2d(&mapW, a.W, a.d_out, a.d_in, a.ldw, kBK, kT)) return cudaErrorInvalidValue;
  } else {   // W stored d_in x d_out: rows = K, columns = N
    if (!make_map_bf16_2d(&mapW, a.W, a.d_in, a.d_out, a.ldw, 64, kBK)) return cudaErrorInvalidValue;
  }
  ProjParams p;
  p.m = static_cast<int>(a.m);
  p.d_in = a.d_in;
  p.d_out = a.d_out;
  p.ldy = a.ldy;
  p.y = reinterpret_cast<__nv_bfloat16*>(a.Y);
  p.status = a.status;
  dim3 grid(a.d_out / kT, static_cast<unsigned>((a.m + kT - 1) / kT));
  cudaError_t e;
  if (wk) {
    e = cudaFuncSetAttribute(proj_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e == cudaSuccess) proj_tc_kernel<true><<<grid, kThreads, kSmemBytes, s>>>(mapA, mapW, mapY, p);
  } else {
    e = cudaFuncSetAttribute(proj_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e == cudaSuccess) proj_tc_kernel<false><<<grid, kThreads, kSmemBytes, s>>>(mapA, mapW, mapY, p);
  }
  if (e != cudaSuccess) return e;
  *n_launched += 1;
  return cudaGetLastError();
}

}  // namespace ispa
