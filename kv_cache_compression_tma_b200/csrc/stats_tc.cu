// stats_tc.cu -- warmup sufficient statistics on tcgen05 tensor cores, sm_100a.
//
// ISPA summary, section 2, stage 2: the closed form dW = (A_loc^T A_loc + lam I)^-1 A_loc^T
// (A_full - A_loc) W needs, per layer, the two d x d factors G = A_loc^T A_loc and
// R = A_loc^T D (D = A_full - A_loc), accumulated over all warmup rows; S = D^T D is added so the
// reconstruction error can be evaluated from statistics alone.  All three are Gram-type products
// X^T Y over the m rows of a chunk, i.e. dense contractions over the row index.
//
// One CTA computes one 128 x 128 output tile of one of G, R, S (blockIdx.z), reducing over all m
// rows in steps of 64.  G and S are symmetric: only tiles on or above the diagonal are computed, and
// each off-diagonal one is also written transposed.  Both operands are the row-major [m, d] activations read as MN-major
// (column index contiguous) tiles by TMA with 128-byte swizzle; the MMA is
// tcgen05.mma.kind::f16 M=128 N=128 K=16 with bf16 operands and an fp32 accumulator in TMEM.
// When the second input is A_full instead of D, the D products are expanded exactly into bf16
// products with negated terms (instruction-descriptor negate bit):
//   R = L^T F - L^T L,   S = F^T F - F^T L - L^T F + L^T L.
// The epilogue stages the fp32 tile in shared memory in the 128-byte-swizzled layout of four
// {32 cols, 128 rows} boxes and adds it into global memory with TMA bulk add-reductions (or bulk
// stores with ISPA_STATS_ZERO), so it never reads the statistics back.
#include <string.h>

#include "gemm_tc.h"
#include "internal.h"
#include "sm100.cuh"

namespace ispa {
namespace {

constexpr int kTile = 128;
constexpr int kBK = 64;                    // rows of X per pipeline stage
constexpr int kSlotBytes = kBK * kTile * 2;  // one operand tile: 64 rows x 128 columns bf16 = 16 KB
constexpr int kBoxBytes = kBK * 128;         // one 64 x 64 box (128-byte rows) = 8 KB
constexpr int kSlots = 4;                    // X1_I, X2_I, X1_J, X2_J
constexpr int kStages = 3;
constexpr int kThreads = 192;
constexpr int kOffBar = kStages * kSlots * kSlotBytes;
constexpr int kOffMisc = kOffBar + (3 * kStages + 1) * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(4 * kTile * 128 <= kOffBar, "the epilogue tile fits in the stage buffers");

__device__ __forceinline__ void fence_proxy_async_smem_stats() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

struct StatsMaps {
  CUtensorMap x1;
  CUtensorMap x2;
  CUtensorMap out[3];  // G, R, S as fp32 {32 cols, 128 rows} boxes
};

__device__ __forceinline__ void bulk_store_2d(const CUtensorMap* map, const void* src, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_add_2d(const CUtensorMap* map, const void* src, int32_t x, int32_t y) {
  asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}

struct Term {
  uint8_t a, b, neg;  // slot indices (0: X1_I, 1: X2_I, 2: X1_J, 3: X2_J), negate flag
};

struct StatsParams {
  int m, d;
  int tiles_per_dim;
  int zero;
  float* out[3];
  int n_terms[3];
  Term terms[3][4];
  uint32_t slot_mask[3];
  unsigned* status;
};

__global__ void __launch_bounds__(kThreads, 1)
    stats_tc_kernel(const __grid_constant__ StatsMaps maps, const StatsParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  volatile int* never = reinterpret_cast<volatile int*>(smem + kOffMisc + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int which = blockIdx.z;  // 0 G, 1 R, 2 S
  const int ti = blockIdx.x / p.tiles_per_dim;
  const int tj = blockIdx.x % p.tiles_per_dim;
  if (which != 1 && tj < ti) return;  // symmetric G, S: the transpose of tile (tj, ti) covers it
  const int n_steps = (p.m + kBK - 1) / kBK;
  const uint32_t mask = p.slot_mask[which];
  uint32_t stage_bytes = 0;
  for (int s = 0; s < kSlots; ++s)
    if (mask & (1u << s)) stage_bytes += kSlotBytes;

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
    tmem_alloc(tmem_slot, kTile);
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
        mbar_arrive_expect_tx(full + s, stage_bytes);
        uint8_t* st = smem + s * kSlots * kSlotBytes;
        for (int slot = 0; slot < kSlots; ++slot) {
          if (!(mask & (1u << slot))) continue;
          const CUtensorMap* map = (slot & 1) ? &maps.x2 : &maps.x1;
          const int col0 = (slot < 2 ? ti : tj) * kTile;
          for (int b = 0; b < 2; ++b)
            tma_load_2d(st + slot * kSlotBytes + b * kBoxBytes, map, full + s, col0 + 64 * b, k * kBK);
        }
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
      const int nt = p.n_terms[which];
      const uint32_t idesc_pos = idesc_bf16_f32(kTile, kTile, true, true, false, false);
      const uint32_t idesc_neg = idesc_bf16_f32(kTile, kTile, true, true, true, false);
      for (int k = 0; k < n_steps; ++k) {
        const int s = k % kStages;
        if (!mbar_wait(full + s, (k / kStages) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t st = smem_u32(smem + s * kSlots * kSlotBytes);
        for (int t = 0; t < nt; ++t) {
          const Term tm = p.terms[which][t];
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = sw128_desc(st + tm.a * kSlotBytes + kk * 16 * 128, kBoxBytes, 1024);
            const uint64_t bd = sw128_desc(st + tm.b * kSlotBytes + kk * 16 * 128, kBoxBytes, 1024);
            const uint32_t acc = (k > 0 || t > 0 || kk > 0) ? 1u : 0u;
            umma_ss(tmem, ad, bd, tm.neg ? idesc_neg : idesc_pos, acc);
          }
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
    // epilogue: thread r owns output row ti*128 + r (TMEM lane r).  The stage buffers are free once
    // the accumulator is complete (every load has been consumed by an MMA).
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const bool ok = mbar_wait_warp(acc_full, 0, never);
    tc_fence_after();
    const bool go = __all_sync(0xffffffffu, ok && !*abort_flag);
    const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const CUtensorMap* om = &maps.out[which];
    const bool mirror = which != 1 && ti != tj;
    for (int pass = 0; pass < (mirror ? 2 : 1); ++pass) {
      if (go) {
#pragma unroll 1
        for (int b = 0; b < kTile / 32; ++b) {
          uint32_t v[32];
          tmem_ld32(taddr + b * 32, v);
          tmem_wait_ld();
          if (pass == 0) {  // row r, columns 32b.. of box b
            uint8_t* row = smem + b * (kTile * 128) + r * 128;
#pragma unroll
            for (int q = 0; q < 8; ++q)
              *reinterpret_cast<float4*>(row + ((q ^ (r & 7)) << 4)) =
                  make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]), __uint_as_float(v[4 * q + 2]),
                              __uint_as_float(v[4 * q + 3]));
          } else {  // transposed: element (r, c) goes to row c, column r (box r / 32)
            uint8_t* box = smem + (r >> 5) * (kTile * 128);
            const int cr = r & 31;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int c = b * 32 + j;
              *reinterpret_cast<float*>(box + c * 128 + ((((cr >> 2) ^ (c & 7))) << 4) + (cr & 3) * 4) =
                  __uint_as_float(v[j]);
            }
          }
        }
        fence_proxy_async_smem_stats();
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");  // the four epilogue warps
      if (go && threadIdx.x == 64) {
        const int orow = (pass == 0 ? ti : tj) * kTile, ocol = (pass == 0 ? tj : ti) * kTile;
        for (int b = 0; b < kTile / 32; ++b) {
          if (p.zero)
            bulk_store_2d(om, smem + b * (kTile * 128), ocol + 32 * b, orow);
          else
            bulk_add_2d(om, smem + b * (kTile * 128), ocol + 32 * b, orow);
        }
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");  // the staging buffer may be reused
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTile);
  }
}

}  // namespace

bool stats_tc_supported(const StatsLaunch& a) {
  if (a.dtype != 0) return false;
  if (a.d % kTile != 0 || a.lda % 8 != 0) return false;
  if (a.m > (1ll << 30)) return false;
  auto al16 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; };
  if (!al16(a.a_loc) || !al16(a.a_second) || !al16(a.G) || !al16(a.R) || !al16(a.S)) return false;
  return true;
}

cudaError_t launch_stats_tc(const StatsLaunch& a, cudaStream_t stream, int* n_launched) {
  StatsMaps maps;
  memset(&maps, 0, sizeof(maps));
  if (!make_map_bf16_2d(&maps.x1, a.a_loc, a.m, a.d, a.lda, 64, kBK)) return cudaErrorInvalidValue;
  if (!make_map_bf16_2d(&maps.x2, a.a_second, a.m, a.d, a.lda, 64, kBK)) return cudaErrorInvalidValue;
  float* outs[3] = {a.G, a.R, a.S};
  for (int w = 0; w < 3; ++w)
    if (!make_map_f32_2d(&maps.out[w], outs[w], a.d, a.d, a.d, 32, kTile, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  StatsParams p;
  memset(&p, 0, sizeof(p));
  p.m = static_cast<int>(a.m);
  p.d = a.d;
  p.tiles_per_dim = a.d / kTile;
  p.zero = a.zero ? 1 : 0;
  p.out[0] = a.G;
  p.out[1] = a.R;
  p.out[2] = a.S;
  p.status = a.status;
  // slots: 0 X1_I (L cols I), 1 X2_I, 2 X1_J, 3 X2_J
  p.n_terms[0] = 1;
  p.terms[0][0] = {0, 2, 0};
  if (!a.second_is_full) {
    p.n_terms[1] = 1;
    p.terms[1][0] = {0, 3, 0};  // L_I^T D_J
    p.n_terms[2] = 1;
    p.terms[2][0] = {1, 3, 0};  // D_I^T D_J
  } else {
    p.n_terms[1] = 2;
    p.terms[1][0] = {0, 3, 0};  // + L_I^T F_J
    p.terms[1][1] = {0, 2, 1};  // - L_I^T L_J
    p.n_terms[2] = 4;
    p.terms[2][0] = {1, 3, 0};  // + F_I^T F_J
    p.terms[2][1] = {1, 2, 1};  // - F_I^T L_J
    p.terms[2][2] = {0, 3, 1};  // - L_I^T F_J
    p.terms[2][3] = {0, 2, 0};  // + L_I^T L_J
  }
  for (int w = 0; w < 3; ++w) {
    uint32_t msk = 0;
    for (int t = 0; t < p.n_terms[w]; ++t) msk |= (1u << p.terms[w][t].a) | (1u << p.terms[w][t].b);
    p.slot_mask[w] = msk;
  }
  cudaError_t e = cudaFuncSetAttribute(stats_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(p.tiles_per_dim * p.tiles_per_dim), 1, 3);
  stats_tc_kernel<<<grid, kThreads, kSmemBytes, stream>>>(maps, p);
  *n_launched += 1;
  return cudaGetLastError();
}

}  // namespace ispa
