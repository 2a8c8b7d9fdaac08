// gemm_tc.cu -- fp32-accurate GEMM on tcgen05 tensor cores for the absorb (split-tf32, sm_100a).
//
// C[M,N] (+)= alpha * op(A)[M,K] op(B)[K,N] with fp32 operands.  Each fp32 value x is split
// into hi = x with its 13 low mantissa bits cleared (exactly a tf32 number) and lo = x - hi (exact in
// fp32); the product is accumulated as hi*hi + hi*lo + lo*hi with tcgen05.mma.kind::tf32 into an fp32
// TMEM accumulator (the lo*lo term is below fp32 resolution).  The tensor core reads a kind::tf32
// operand's 32-bit element by its top 19 bits, i.e. it truncates x to hi by itself: the staged fp32
// tile serves as hi unchanged and only lo is written (measured on B200: dW of the absorb bit-identical
// with and without clearing the low bits in shared memory first, at d = 256, 1536 and 3072).  An operand known to hold tf32 numbers
// (a widened bf16 weight) has lo = 0: its split and its lo products are skipped.  This keeps the absorb's fp32 accuracy
// (B = R W, S W, the Cholesky panel / trailing updates and the triangular-solve GEMMs) at tensor-core
// speed instead of CUDA-core FFMA.
//
// One CTA computes one 128 x BN tile of C, BN = 128 (3-stage ring) or 256 (2-stage ring, for the
// large products: each staged A byte then feeds twice the work, which matters because the operand
// splits and the MMAs share the shared-memory bandwidth).  Warp roles
// (192 threads):
//   warp 0      TMA producer: K chunks of 32 of the A and B tiles, 128-byte swizzle
//   warp 1      TMEM owner + single-thread MMA issuer (3 MMAs of K = 8 per 8 columns of K)
//   warps 2..5  write lo = x - hi of the landed fp32 tiles into the second buffer, then run the
//               epilogue (thread = row = TMEM lane): C = alpha * acc or C += alpha * acc.
// Operand majorness follows from the storage: op(A) = A is K-major, op(A) = A^T is MN-major; op(B) =
// B is MN-major, op(B) = B^T is K-major.  The absorb hands in tensor maps over whole matrices plus
// the sub-block origin; every extent is a multiple of 128 on this path (d % 128 == 0).  The result
// leaves through TMA bulk stores: C = alpha * op(A) op(B), or C += alpha * op(A) op(B) by bulk
// add-reduction (the absorb's trailing updates), so the epilogue never reads C.
#include <string.h>

#include <type_traits>

#include "gemm_tc.h"
#include "internal.h"
#include "sm100.cuh"

namespace ispa {
namespace {

constexpr int kT = 128;         // tile M (and the N granularity)
constexpr int kBK = 32;         // K per stage (one 128-byte swizzle row of fp32)
constexpr int kTileBytes = kT * kBK * 4;  // 16 KB: one 128 x 32 fp32 operand tile
constexpr int kThreads = 192;

// Stage layout: A [, A_lo], B [, B_lo]; an operand that is exact in tf32 (EX bit 0: A, bit 1: B) has
// no lo buffer, so its stages are smaller and the ring deeper for the same shared memory (the
// single-product W W^T runs four stages of 128 x 256 tiles, and its loads stay in flight longer).
template <int BN, int EX>
struct GCfg {
  static constexpr int kBBytes = BN * kBK * 4;  // one B tile
  static constexpr int kOffALo = kTileBytes;
  static constexpr int kOffB = (EX & 1) ? kTileBytes : 2 * kTileBytes;
  static constexpr int kOffBLo = kOffB + kBBytes;
  static constexpr int kStageBytes = kOffB + ((EX & 2) ? 1 : 2) * kBBytes;
  static constexpr int kRing = 196608;  // bytes of stages (leaves room below the 227 KB limit)
  static constexpr int kStages = kRing / kStageBytes > 6 ? 6 : kRing / kStageBytes;
  static constexpr int kOffBar = kStages * kStageBytes;
  static constexpr int kOffMisc = kOffBar + (3 * kStages + 1) * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kStages * kStageBytes >= (BN / 32) * kTileBytes, "epilogue staging fits the ring");
};

// kind::tf32 instruction descriptor: D f32, A/B tf32 (format 2), majors, N >> 3, M >> 4
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (2u << 7) | (2u << 10) | (a_mn ? (1u << 15) : 0u) | (b_mn ? (1u << 16) : 0u) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void umma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Shared-memory descriptor of an MN-major 32-bit operand: 128-byte rows along M/N whose 32-byte
// chunks are swizzled with a 4-row period (layout type 1; the TMA writes it with
// CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B).  LBO = stride between 32-element MN chunks, SBO = stride
// between 4-row K groups.
__device__ __forceinline__ uint64_t sw128_32b_desc(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFF) << 32;
  d |= 1ull << 46;
  d |= 1ull << 61;
  return d;
}

__device__ __forceinline__ uint64_t operand_desc(bool mn_major, uint32_t addr) {
  // K-major: 128-byte swizzle, 8-row groups 1024 bytes apart; MN-major: 32-byte-atom swizzle,
  // 32-element chunks 4 KB apart (one {32 x 32} box each), 4-row groups 512 bytes apart
  return mn_major ? sw128_32b_desc(addr, kTileBytes / 4, 512) : sw128_desc(addr, 16, 1024);
}

// 2-D tiled bulk tensor store (shared -> global) or add-reduction into global, bulk-group completion.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(smem_src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, const void* smem_src, int32_t x,
                                                  int32_t y) {
  asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(smem_src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

struct GemmParams {
  int M, N, K;
  int a_r0, a_c0;  // origin of op(A)'s storage block in A's tensor map (row, column)
  int b_r0, b_c0;
  int c_r0, c_c0;  // origin of C's block in C's tensor map
  float alpha;
  int accumulate;  // 0: C = alpha * acc (bulk store); 1: C += alpha * acc (bulk add-reduction)
  int lower_only;
  int exact;       // bit 0: A's values are tf32 numbers (a widened bf16 matrix), bit 1: B's; lo part zero
  unsigned* status;
};

template <bool A_MN, bool B_MN, int BN, int EX>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                   const __grid_constant__ CUtensorMap mapC, const GemmParams p) {
  using G = GCfg<BN, EX>;
  constexpr int kStages = G::kStages;
  constexpr int kStageBytes = G::kStageBytes;
  const int tm = blockIdx.y, tn = blockIdx.x;
  const int m0 = tm * kT, n0 = tn * BN;
  if (p.lower_only && n0 > m0 + kT - 1) return;  // tile strictly above the diagonal: nothing to do
  griddep_launch_dependents();

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + G::kOffBar);
  uint64_t* conv = full + kStages;
  uint64_t* empty = conv + kStages;
  uint64_t* acc_full = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + G::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + G::kOffMisc + 4);
  volatile int* never = reinterpret_cast<volatile int*>(smem + G::kOffMisc + 8);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_steps = p.K / kBK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(full + i, 1);
      mbar_init(conv + i, 4);  // one arrival per split warp
      mbar_init(empty + i, 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    *never = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();  // operands and C are written by the previous grid of the stream (PDL launches)

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
        mbar_arrive_expect_tx(full + s, kTileBytes + G::kBBytes);
        const int kk = k * kBK;
        if (!A_MN) {  // A stored M x K: box {32 (K), 128 (M rows)}
          tma_load_2d(st, &mapA, full + s, p.a_c0 + kk, p.a_r0 + m0);
        } else {  // A stored K x M: four boxes {32 (M), 32 (K rows)}
          for (int b = 0; b < 4; ++b)
            tma_load_2d(st + b * (kTileBytes / 4), &mapA, full + s, p.a_c0 + m0 + 32 * b, p.a_r0 + kk);
        }
        uint8_t* sb = st + G::kOffB;
        if (!B_MN) {  // B stored N x K: boxes {32 (K), 128 (N rows)}, contiguous along N
          for (int h = 0; h < BN / kT; ++h)
            tma_load_2d(sb + h * kTileBytes, &mapB, full + s, p.b_c0 + kk, p.b_r0 + n0 + kT * h);
        } else {  // B stored K x N: boxes {32 (N), 32 (K rows)}, 4 KB apart
          for (int b = 0; b < BN / 32; ++b)
            tma_load_2d(sb + b * (kTileBytes / 4), &mapB, full + s, p.b_c0 + n0 + 32 * b, p.b_r0 + kk);
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
      const uint32_t idesc = idesc_tf32(kT, BN, A_MN, B_MN);
      for (int k = 0; k < n_steps; ++k) {
        const int s = k % kStages;
        if (!mbar_wait(conv + s, (k / kStages) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_hi = smem_u32(smem + s * kStageBytes);
        const uint32_t a_lo = a_hi + G::kOffALo;  // used only when A is split
        const uint32_t b_hi = a_hi + G::kOffB;
        const uint32_t b_lo = a_hi + G::kOffBLo;  // used only when B is split
#pragma unroll
        for (int kk = 0; kk < kBK / 8; ++kk) {
          // K-major: 8 fp32 = 32 bytes along the swizzled row; MN-major: 8 K rows = one 1024-byte group
          const uint32_t ao = A_MN ? kk * 1024 : kk * 32;
          const uint32_t bo = B_MN ? kk * 1024 : kk * 32;
          const uint64_t ah = operand_desc(A_MN, a_hi + ao), al = operand_desc(A_MN, a_lo + ao);
          const uint64_t bh = operand_desc(B_MN, b_hi + bo), bl = operand_desc(B_MN, b_lo + bo);
          const uint32_t acc0 = (k > 0 || kk > 0) ? 1u : 0u;
          umma_tf32(tmem, ah, bh, idesc, acc0);
          if (!((p.exact | EX) & 2)) umma_tf32(tmem, ah, bl, idesc, 1u);
          if (!((p.exact | EX) & 1)) umma_tf32(tmem, al, bh, idesc, 1u);
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
    // split warps: lo into the second buffer (the staged tile itself is hi to the MMA), for the A and
    // the B tile of each stage
    const int t = threadIdx.x - 64;  // 0..127
    bool ok = true;
    for (int k = 0; k < n_steps; ++k) {
      const int s = k % kStages;
      if (!mbar_wait_warp(full + s, (k / kStages) & 1, abort_flag)) {  // warp-uniform: one arrival per warp
        ok = false;
        break;
      }
      uint8_t* st = smem + s * kStageBytes;
      for (int which = 0; which < 2; ++which) {
        if ((p.exact | EX) & (1 << which)) continue;  // an exact operand needs no split
        const int bytes = which ? G::kBBytes : kTileBytes;
        const float4* x = reinterpret_cast<const float4*>(st + (which ? G::kOffB : 0));
        float4* lo = reinterpret_cast<float4*>(st + (which ? G::kOffBLo : G::kOffALo));
#pragma unroll 8
        for (int i = 0; i < bytes / 16 / 128; ++i) {
          const int idx = t + 128 * i;
          float4 v = x[idx], h, l;
          h.x = __uint_as_float(__float_as_uint(v.x) & 0xFFFFE000u);
          h.y = __uint_as_float(__float_as_uint(v.y) & 0xFFFFE000u);
          h.z = __uint_as_float(__float_as_uint(v.z) & 0xFFFFE000u);
          h.w = __uint_as_float(__float_as_uint(v.w) & 0xFFFFE000u);
          l.x = v.x - h.x;
          l.y = v.y - h.y;
          l.z = v.z - h.z;
          l.w = v.w - h.w;
          lo[idx] = l;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(conv + s);  // one arrival per warp, after every lane's stores
    }
    if (!ok) {
      atomicOr(p.status, kStatusTimeout);
      *abort_flag = 1;
    }
    // epilogue: TMEM -> shared memory in the 128-byte-swizzled layout of four {32 cols, 128 rows}
    // boxes -> one bulk tensor store (C = alpha acc) or add-reduction (C += alpha acc) per box.  The
    // stage buffers are free: every MMA, hence every load, has completed when acc_full fires.  Tiles
    // on the diagonal of a lower-only update are written whole (the strict upper triangle of such an
    // output is never read).
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const bool done = mbar_wait_warp(acc_full, 0, never);
    tc_fence_after();
    const bool go = __all_sync(0xffffffffu, done && !*abort_flag);
    if (go) {
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll 1
      for (int b = 0; b < BN / 32; ++b) {
        uint32_t v[32];
        tmem_ld32(taddr + b * 32, v);
        tmem_wait_ld();
        uint8_t* row = smem + b * kTileBytes + r * 128;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float4 o = make_float4(p.alpha * __uint_as_float(v[4 * q]), p.alpha * __uint_as_float(v[4 * q + 1]),
                                 p.alpha * __uint_as_float(v[4 * q + 2]), p.alpha * __uint_as_float(v[4 * q + 3]));
          *reinterpret_cast<float4*>(row + ((q ^ (r & 7)) << 4)) = o;
        }
      }
      fence_proxy_async_smem();
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");  // the four epilogue warps
    if (go && threadIdx.x == 64) {
      for (int b = 0; b < BN / 32; ++b) {
        if (p.accumulate)
          tma_reduce_add_2d(&mapC, smem + b * kTileBytes, p.c_c0 + n0 + 32 * b, p.c_r0 + m0);
        else
          tma_store_2d(&mapC, smem + b * kTileBytes, p.c_c0 + n0 + 32 * b, p.c_r0 + m0);
      }
      bulk_commit();
      bulk_wait_read0();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}

}  // namespace

bool make_map_f32_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                     uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 4};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_operand_maps(F32Operand* op, const float* base, uint64_t rows, uint64_t cols, uint64_t ld) {
  op->base = base;
  return make_map_f32_2d(&op->kmajor, base, rows, cols, ld, kBK, kT, CU_TENSOR_MAP_SWIZZLE_128B) &&
         make_map_f32_2d(&op->mnmajor, base, rows, cols, ld, 32, kBK, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B);
}

cudaError_t gemm_tc(bool ta, bool tb, int M, int N, int K, float alpha, const F32Operand& A, int a_r0, int a_c0,
                    const F32Operand& B, int b_r0, int b_c0, bool accumulate, const F32Operand& C, int c_r0, int c_c0,
                    bool lower_only, unsigned* status, cudaStream_t s, int* n_launched, bool pdl, int exact) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  if (M % kT || N % kT || K % kBK || K <= 0) return cudaErrorInvalidValue;
  GemmParams p;
  p.M = M;
  p.N = N;
  p.K = K;
  p.a_r0 = a_r0;
  p.a_c0 = a_c0;
  p.b_r0 = b_r0;
  p.b_c0 = b_c0;
  p.c_r0 = c_r0;
  p.c_c0 = c_c0;
  p.alpha = alpha;
  p.accumulate = accumulate ? 1 : 0;
  p.lower_only = lower_only ? 1 : 0;
  p.exact = exact & 3;
  p.status = status;
  // op(A) = A (M x K stored) -> K-major; op(A) = A^T (stored K x M) -> MN-major
  const CUtensorMap& ma = ta ? A.mnmajor : A.kmajor;
  // op(B) = B (stored K x N) -> MN-major; op(B) = B^T (stored N x K) -> K-major
  const CUtensorMap& mb = tb ? B.kmajor : B.mnmajor;
  const CUtensorMap& mc = C.kmajor;  // {32 cols, 128 rows} boxes, 128-byte swizzle
  // 128 x 256 tiles whenever there are enough of them to keep most SMs busy: one wide tile does the
  // work of two narrow ones at about 1.3x less time, so it pays from about half a wave of wide tiles
  // on.  A lower-triangle update runs about half its tiles; its wide tiles on the diagonal also write
  // part of the strict upper triangle, which no caller reads.
  const long long wide_tiles = static_cast<long long>(M / kT) * (N / 256);
  const long long wide_active = lower_only ? (wide_tiles + M / kT) / 2 : wide_tiles;
  const bool wide = N % 256 == 0 && wide_active >= 80;
  dim3 grid(N / (wide ? 256 : kT), M / kT);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  // the layout instance: both operands exact, B exact, or the general one (which also serves an
  // exact A alone through the runtime flag)
  const int ex = (p.exact == 3) ? 3 : (p.exact == 2 ? 2 : 0);
  auto launch = [&](auto kernel, int smem_bytes) -> cudaError_t {
    cfg.dynamicSmemBytes = smem_bytes;
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
    if (err != cudaSuccess) return err;
    return cudaLaunchKernelEx(&cfg, kernel, ma, mb, mc, p);
  };
  auto by_ex = [&](auto tag_amn, auto tag_bmn, auto tag_bn) -> cudaError_t {
    constexpr bool AM = decltype(tag_amn)::value, BM = decltype(tag_bmn)::value;
    constexpr int BNv = decltype(tag_bn)::value;
    if (ex == 3) return launch(gemm_tc_kernel<AM, BM, BNv, 3>, GCfg<BNv, 3>::kSmemBytes);
    if (ex == 2) return launch(gemm_tc_kernel<AM, BM, BNv, 2>, GCfg<BNv, 2>::kSmemBytes);
    return launch(gemm_tc_kernel<AM, BM, BNv, 0>, GCfg<BNv, 0>::kSmemBytes);
  };
  using T_ = std::true_type;
  using F_ = std::false_type;
  using N256 = std::integral_constant<int, 256>;
  using N128 = std::integral_constant<int, 128>;
  cudaError_t e;
  if (!ta && !tb)
    e = wide ? by_ex(F_{}, T_{}, N256{}) : by_ex(F_{}, T_{}, N128{});
  else if (!ta && tb)
    e = wide ? by_ex(F_{}, F_{}, N256{}) : by_ex(F_{}, F_{}, N128{});
  else if (ta && !tb)
    e = wide ? by_ex(T_{}, T_{}, N256{}) : by_ex(T_{}, T_{}, N128{});
  else
    e = wide ? by_ex(T_{}, F_{}, N256{}) : by_ex(T_{}, F_{}, N128{});
  if (e != cudaSuccess) return e;
  *n_launched += 1;
  return cudaGetLastError();
}

}  // namespace ispa
