// stats_tc.cu -- warmup sufficient statistics on tcgen05 tensor cores, sm_100a.
//
// ISPA summary, section 2, stage 2: the closed form dW = (A_loc^T A_loc + lam I)^-1 A_loc^T
// (A_full - A_loc) W needs, per layer, the two d x d factors G = A_loc^T A_loc and
// R = A_loc^T D (D = A_full - A_loc), accumulated over all warmup rows; S = D^T D is added so the
// reconstruction error can be evaluated from statistics alone.  Together they are the Gram matrix of
// X = [A_loc | D] (m x 2d):  X^T X = [[G, R], [R^T, S]], a dense contraction over the row index.
//
// One CTA computes one 256 x 256 block of that Gram: for 128-column slabs I <= J of the d columns it
// stages L_I, D_I, L_J, D_J (64 rows per pipeline stage, all four used) and accumulates four
// 128 x 128 products in TMEM (all 512 columns):
//     G_IJ = L_I^T L_J,   R_IJ = L_I^T D_J,   R_JI^T = D_I^T L_J,   S_IJ = D_I^T D_J,
// so every staged byte feeds two products (twice the operand reuse of one product per tile).  The
// slabs L_J and D_J sit next to each other in shared memory, so each pair of products with the same
// A operand is one tcgen05.mma.kind::f16 of M=128 N=256 K=16 (B = [L_J | D_J]): [G_IJ | R_IJ] and
// [R_JI^T | S_IJ].  Against four N=128 MMAs this reads a quarter fewer shared-memory bytes per flop
// and issues half the instructions.  On the diagonal (I == J) two slabs are staged and [G_II | R_II]
// (N=256) and S_II (N=128) formed.  G and S are symmetric: the off-diagonal blocks are also written
// transposed, and R_JI^T is written transposed into R's block (J, I).  Operands are the row-major
// [m, d] activations read as MN-major (column index contiguous) tiles by TMA with 128-byte swizzle;
// bf16 operands, fp32 accumulators.
// When the second input is A_full (F) instead of D, the D products are expanded exactly into bf16
// products with negated terms (instruction-descriptor negate bit), one N=128 MMA per term:
//   R = L^T F - L^T L,   S = F^T F - F^T L - L^T F + L^T L.
// For narrow layers the row range is split over several CTAs per block (more CTAs than blocks).
// The epilogue stages each fp32 tile in shared memory in the 128-byte-swizzled layout of four
// {32 cols, 128 rows} boxes (three staging buffers in rotation) and adds it into global memory with
// TMA bulk add-reductions (bulk stores with ISPA_STATS_ZERO and one row range), so it never reads
// the statistics back.
#include <string.h>

#include "gemm_tc.h"
#include "internal.h"
#include "sm100.cuh"

namespace ispa {
namespace {

constexpr int kTile = 128;
constexpr int kBK = 64;                      // rows of X per pipeline stage
constexpr int kSlotBytes = kBK * kTile * 2;  // one operand slab: 64 rows x 128 columns bf16 = 16 KB
constexpr int kBoxBytes = kBK * 128;         // one 64 x 64 box (128-byte rows) = 8 KB
constexpr int kSlots = 4;                    // L_I, X2_I, L_J, X2_J
constexpr int kStages = 3;
constexpr int kThreads = 192;
constexpr int kOutTileBytes = kTile * kTile * 4;  // one fp32 output tile (four 32-column boxes)
constexpr int kOffBar = kStages * kSlots * kSlotBytes;
constexpr int kOffMisc = kOffBar + (3 * kStages + 1) * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(3 * kOutTileBytes <= kOffBar, "three epilogue tiles fit in the stage buffers");

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
  uint8_t a, b, neg;  // slot indices (0: L_I, 1: X2_I, 2: L_J, 3: X2_J), negate flag
};

// Accumulators: 0 G_IJ, 1 R_IJ, 2 R_JI (R_JI^T with `fused`), 3 S_IJ (TMEM columns 128 * index).
struct StatsParams {
  int m, d;
  int n_slabs;     // d / 128
  int n_split;     // row ranges per block
  int rows_split;  // rows per range (a multiple of kBK)
  int store;       // 1: bulk stores (zero-fill semantics), 0: bulk add-reductions
  int fused;       // second input D: [G_IJ | R_IJ] and [R_JI^T | S_IJ] as two N = 256 products
  int n_terms[4];
  Term terms[4][4];
  unsigned* status;
};

// Block index -> slabs (I, J), I <= J, row-major over the upper triangle.
__device__ __forceinline__ void block_slabs(int idx, int n, int& I, int& J) {
  int i = 0, rem = idx;
  while (rem >= n - i) {
    rem -= n - i;
    ++i;
  }
  I = i;
  J = i + rem;
}

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
  int I, J;
  block_slabs(blockIdx.x, p.n_slabs, I, J);
  const bool diag = I == J;
  const int row0 = blockIdx.y * p.rows_split;
  const int row1 = min(p.m, row0 + p.rows_split);
  const int n_steps = row1 > row0 ? (row1 - row0 + kBK - 1) / kBK : 0;
  const int n_slots = diag ? 2 : 4;  // on the diagonal slots 2, 3 are slots 0, 1
  const uint32_t stage_bytes = n_slots * kSlotBytes;

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
    tmem_alloc(tmem_slot, 512);
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
        for (int slot = 0; slot < n_slots; ++slot) {
          const CUtensorMap* map = (slot & 1) ? &maps.x2 : &maps.x1;
          const int col0 = (slot < 2 ? I : J) * kTile;
          for (int b = 0; b < 2; ++b)
            tma_load_2d(st + slot * kSlotBytes + b * kBoxBytes, map, full + s, col0 + 64 * b, row0 + k * kBK);
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
      const uint32_t idesc_pos = idesc_bf16_f32(kTile, kTile, true, true, false, false);
      const uint32_t idesc_neg = idesc_bf16_f32(kTile, kTile, true, true, true, false);
      const uint32_t idesc_wide = idesc_bf16_f32(kTile, 2 * kTile, true, true, false, false);
      for (int k = 0; k < n_steps; ++k) {
        const int s = k % kStages;
        if (!mbar_wait(full + s, (k / kStages) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t st = smem_u32(smem + s * kSlots * kSlotBytes);
        if (p.fused) {
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint32_t accum = (k > 0 || kk > 0) ? 1u : 0u;
            const uint64_t a0 = sw128_desc(st + kk * 16 * 128, kBoxBytes, 1024);
            const uint64_t a1 = sw128_desc(st + kSlotBytes + kk * 16 * 128, kBoxBytes, 1024);
            // B = [L_J | D_J] (on the diagonal [L_I | D_I]): four 64-column chunks kBoxBytes apart
            const uint64_t bw = sw128_desc(st + (diag ? 0 : 2) * kSlotBytes + kk * 16 * 128, kBoxBytes, 1024);
            umma_ss(tmem, a0, bw, idesc_wide, accum);  // [G_IJ | R_IJ]
            if (!diag) {
              umma_ss(tmem + 2 * kTile, a1, bw, idesc_wide, accum);  // [R_JI^T | S_IJ]
            } else {
              const uint64_t b1 = sw128_desc(st + kSlotBytes + kk * 16 * 128, kBoxBytes, 1024);
              umma_ss(tmem + 3 * kTile, a1, b1, idesc_pos, accum);  // S_II
            }
          }
          umma_commit(empty + s);
          continue;
        }
        for (int acc = 0; acc < 4; ++acc) {
          if (diag && acc == 2) continue;  // R_JI is R_IJ on the diagonal
          for (int t = 0; t < p.n_terms[acc]; ++t) {
            const Term tm = p.terms[acc][t];
            const int sa = diag ? (tm.a & 1) : tm.a, sb = diag ? (tm.b & 1) : tm.b;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint64_t ad = sw128_desc(st + sa * kSlotBytes + kk * 16 * 128, kBoxBytes, 1024);
              const uint64_t bd = sw128_desc(st + sb * kSlotBytes + kk * 16 * 128, kBoxBytes, 1024);
              const uint32_t accum = (k > 0 || t > 0 || kk > 0) ? 1u : 0u;
              umma_ss(tmem + acc * kTile, ad, bd, tm.neg ? idesc_neg : idesc_pos, accum);
            }
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
    // epilogue: thread r owns row r of every accumulator (TMEM lane r).  The stage buffers are free
    // once the accumulators are complete (every load has been consumed by an MMA).
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const bool ok = mbar_wait_warp(acc_full, 0, never);
    tc_fence_after();
    const bool go = __all_sync(0xffffffffu, ok && !*abort_flag) && n_steps > 0;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    // outputs: (accumulator, matrix, tile row, tile column, transposed)
    int n_out = 0;
    int o_acc[6], o_mat[6], o_row[6], o_col[6], o_tr[6];
    auto add_out = [&](int acc, int mat, int tr_, int tc_, int tr) {
      o_acc[n_out] = acc;
      o_mat[n_out] = mat;
      o_row[n_out] = tr_;
      o_col[n_out] = tc_;
      o_tr[n_out] = tr;
      ++n_out;
    };
    add_out(0, 0, I, J, 0);
    add_out(1, 1, I, J, 0);
    add_out(3, 2, I, J, 0);
    if (!diag) {
      add_out(2, 1, J, I, p.fused ? 1 : 0);
      add_out(0, 0, J, I, 1);
      add_out(3, 2, J, I, 1);
    }
    for (int o = 0; o < n_out; ++o) {
      uint8_t* buf = smem + (o % 3) * kOutTileBytes;
      if (o >= 3) {
        // the buffer's previous tile must have been read by its bulk operation
        if (threadIdx.x == 64) asm volatile("cp.async.bulk.wait_group.read 2;" ::: "memory");
        asm volatile("bar.sync 1, 128;" ::: "memory");
      }
      if (go) {
        const uint32_t taddr = tmem + lane_addr + o_acc[o] * kTile;
#pragma unroll 1
        for (int b = 0; b < kTile / 32; ++b) {
          uint32_t v[32];
          tmem_ld32(taddr + b * 32, v);
          tmem_wait_ld();
          if (!o_tr[o]) {  // row r, columns 32b.. of box b
            uint8_t* row = buf + b * (kTile * 128) + r * 128;
#pragma unroll
            for (int q = 0; q < 8; ++q)
              *reinterpret_cast<float4*>(row + ((q ^ (r & 7)) << 4)) =
                  make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]), __uint_as_float(v[4 * q + 2]),
                              __uint_as_float(v[4 * q + 3]));
          } else {  // transposed: element (r, c) goes to row c, column r (box r / 32)
            uint8_t* box = buf + (r >> 5) * (kTile * 128);
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
        const CUtensorMap* om = &maps.out[o_mat[o]];
        const int orow = o_row[o] * kTile, ocol = o_col[o] * kTile;
        for (int b = 0; b < kTile / 32; ++b) {
          if (p.store)
            bulk_store_2d(om, buf + b * (kTile * 128), ocol + 32 * b, orow);
          else
            bulk_add_2d(om, buf + b * (kTile * 128), ocol + 32 * b, orow);
        }
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      }
    }
    if (threadIdx.x == 64) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
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
  p.n_slabs = a.d / kTile;
  p.status = a.status;
  const int n_blocks = p.n_slabs * (p.n_slabs + 1) / 2;
  // Split the rows over several CTAs per block when the blocks alone leave SMs idle: pick the split
  // (at most 8) that minimises waves x (rows per CTA), with at least 8 pipeline steps per CTA.
  int sms = 148;
  {
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  const long long steps_total = (a.m + kBK - 1) / kBK;
  int best = 1;
  double best_cost = 1e30;
  for (int s = 1; s <= 8; ++s) {
    const long long steps = (steps_total + s - 1) / s;
    if (s > 1 && steps < 8) break;
    const long long ctas = static_cast<long long>(n_blocks) * s;
    const double cost = static_cast<double>((ctas + sms - 1) / sms) * (steps + 6);  // + epilogue, in steps
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = s;
    }
  }
  p.n_split = best;
  p.rows_split = static_cast<int>(((steps_total + best - 1) / best) * kBK);
  // overwriting (ISPA_STATS_ZERO) with several row ranges per block: zero first, then add
  if (a.zero && best > 1) {
    const size_t bytes = sizeof(float) * static_cast<size_t>(a.d) * a.d;
    for (int w = 0; w < 3; ++w) {
      cudaError_t e = cudaMemsetAsync(outs[w], 0, bytes, stream);
      if (e != cudaSuccess) return e;
    }
  }
  p.store = (a.zero && best == 1) ? 1 : 0;
  // slots: 0 L_I, 1 X2_I, 2 L_J, 3 X2_J;  accumulators: 0 G_IJ, 1 R_IJ, 2 R_JI, 3 S_IJ
  p.n_terms[0] = 1;
  p.terms[0][0] = {0, 2, 0};  // L_I^T L_J
  if (!a.second_is_full) {
    p.fused = 1;  // the MMA loop forms these four products as two N = 256 MMAs; the terms are unused
    p.n_terms[1] = 1;
    p.terms[1][0] = {0, 3, 0};  // L_I^T D_J
    p.n_terms[2] = 1;
    p.terms[2][0] = {2, 1, 0};  // L_J^T D_I
    p.n_terms[3] = 1;
    p.terms[3][0] = {1, 3, 0};  // D_I^T D_J
  } else {
    p.n_terms[1] = 2;
    p.terms[1][0] = {0, 3, 0};  // + L_I^T F_J
    p.terms[1][1] = {0, 2, 1};  // - L_I^T L_J
    p.n_terms[2] = 2;
    p.terms[2][0] = {2, 1, 0};  // + L_J^T F_I
    p.terms[2][1] = {2, 0, 1};  // - L_J^T L_I
    p.n_terms[3] = 4;
    p.terms[3][0] = {1, 3, 0};  // + F_I^T F_J
    p.terms[3][1] = {1, 2, 1};  // - F_I^T L_J
    p.terms[3][2] = {0, 3, 1};  // - L_I^T F_J
    p.terms[3][3] = {0, 2, 0};  // + L_I^T L_J
  }
  cudaError_t e = cudaFuncSetAttribute(stats_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(n_blocks), static_cast<unsigned>(best), 1);
  stats_tc_kernel<<<grid, kThreads, kSmemBytes, stream>>>(maps, p);
  *n_launched += 1;
  return cudaGetLastError();
}

}  // namespace ispa
