// attn_tc.cu -- decomposable (dual-stream) attention on tcgen05 tensor cores, sm_100a.
//
// ISPA summary, section 2, stage 1 ("Decomposable Attention"): one pass over the KV cache yields
// both A_loc (sink + current chunk) and A_full (sink + current chunk + history) by keeping the
// online-softmax state of the two key branches apart and merging them post-hoc by log-sum-exp.
//
// One CTA computes two 128-query-row tiles (A and B) of one head.  Keys are walked once, in the
// order sink tiles, local tiles (the local branch), history tiles (the history branch), 128 keys per
// tile; both query tiles consume the same K/V tiles, so each K/V byte staged in shared memory feeds
// 256 query rows.  The tensor core alternates between the two tiles, so that one tile's softmax runs
// while the other tile's products are computed (ping-pong):
//     ... PV_A(j)  S_A(j+1)  PV_B(j)  S_B(j+1)  PV_A(j+1) ...
// with S_X(j) = Q_X K_j^T (SS MMA into TMEM) and O_X += P_X(j) V_j (TS MMA: P read from TMEM).
//
// Branch bookkeeping per query row (one thread per row): a shared running max m (log2 units), the
// local sum l_loc and the history sum l_hist, and ONE fp32 accumulator O in TMEM.  At the branch
// switch (the first history tile) O holds the local branch alone: it is normalised and written out
// as O_loc (with lse_loc), and -- when D is requested -- its fp32 values are parked in the row's own
// O_full and D output slots (exactly 4 bytes per element between them).  The history tiles then
// accumulate into the same O, so at the end
//     O_full = O / (l_loc + l_hist),   D = O_full - O_loc (fp32, from the parked values),
//     lse_loc = m_switch + log2 l_loc(switch),   lse_hist = m + log2 l_hist,
// which is sigma(lse_loc - lse_hist) O_loc + sigma(lse_hist - lse_loc) O_hist.  Without history
// O_full is the same bf16 values as O_loc and D is zero.  The running max is raised (and O, l
// rescaled) only when a tile's maximum exceeds it by more than 2^8.
//
// Warp roles (320 threads):
//   warps 0..3  softmax + epilogue of query tile A, warps 4..7 of tile B: thread = query row =
//               TMEM lane; each thread loads its 128 scores, writes P = exp2(S*scale*log2e - m) as
//               bf16 over the first 64 columns of the same TMEM buffer; a share of the exponentials
//               runs as a cubic on the FMA pipe (per key tile the MUFU unit alone needs as many
//               cycles as the tensor core);
//   warp 8      TMA producer: both Q tiles once, then K_0, V_0, K_1, V_1, ... through a ring of slots;
//   warp 9      TMEM owner + single-thread MMA issuer.
// TMEM columns: [0,128) S/P of tile A, [128,256) S/P of tile B, then O_A and O_B (HD columns each).
// Every barrier wait is bounded (see sm100.cuh); a timeout records ISPA_ERR_TIMEOUT and unwinds.
#include <math.h>
#include <string.h>

#include "../../include/ispa.h"
#include "internal.h"
#include "sm100.cuh"

namespace ispa {
namespace {

constexpr int kBM = 128;   // query rows per tile (two tiles per CTA)
constexpr int kBN = 128;   // keys per tile
constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Columns (of the 128 of a full key tile) whose exponentials run on the FMA pipe, not the MUFU unit
// (a multiple of 16; a build-time tuning constant).
#ifndef ISPA_ATTN_POLY_COLS
#define ISPA_ATTN_POLY_COLS 32
#endif
constexpr int kPolyCols = ISPA_ATTN_POLY_COLS;
static_assert(kPolyCols % 16 == 0 && kPolyCols <= 128, "poly columns");

struct AttnMaps {
  CUtensorMap q;
  CUtensorMap k[3];
  CUtensorMap v[3];
};

struct AttnParams {
  int n_q;
  int n_kv[3];
  int tiles[3];
  float scale_log2;
  void* o_loc;
  void* o_full;
  void* d_out;
  long long ld_o;
  float* lse_loc;
  float* lse_hist;
  unsigned* status;
  uint32_t test_flags;
  const float* bias[3];  // optional per-key logit bias of each segment, [n_heads, n_kv] (natural log)
  long long ld_bias[3];
};

template <int HD>
struct Cfg {
  static constexpr int kBoxes = HD / 64;            // 128-byte boxes per row
  static constexpr int kBoxBytes = 128 * 128;       // one 64-column box of 128 rows
  static constexpr int kQBytes = kBM * HD * 2;      // one query tile
  static constexpr int kSlotBytes = kBN * HD * 2;   // one K or V tile
  static constexpr int kSlots = (HD == 128) ? 5 : 8;
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = 2 * kQBytes;
  static constexpr int kOffBar = kOffKV + kSlots * kSlotBytes;
  // barriers: q_full, full[slots], empty[slots], s_full[2], p_ready[2], o_final, final
  static constexpr int kNumBars = 1 + 2 * kSlots + 2 + 2 + 1 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16;  // base is 1024-byte aligned
  static constexpr uint32_t kColO = 256;            // O_A at 256, O_B at 256 + HD
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, kBN, false, false);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, HD, false, true);
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kColO + 2 * HD <= 512, "TMEM budget");
};

__device__ __forceinline__ void tile_info(const AttnParams& p, int t, int& seg, int& key0, int& valid) {
  const int t0 = p.tiles[0], t1 = t0 + p.tiles[1];
  if (t < t0) {
    seg = 0;
    key0 = t * kBN;
  } else if (t < t1) {
    seg = 1;
    key0 = (t - t0) * kBN;
  } else {
    seg = 2;
    key0 = (t - t1) * kBN;
  }
  valid = min(kBN, p.n_kv[seg] - key0);
}

// 2^x without the MUFU unit, for x in [-126, 64]: x = j + f with j = round(x) (adding 1.5 * 2^23
// leaves j in the low mantissa bits) and f in [-1/2, 1/2]; 2^f is a cubic fitted to it on that
// interval (least squares with Lawson reweighting toward the minimax relative error: 7.7e-5 at most,
// far below the bf16 rounding of P); 2^j is added to the exponent field.  Two at a time on the
// f32x2 pipes.
constexpr float kExpC0 = 0.99992758f, kExpC1 = 0.69325161f, kExpC2 = 0.242615268f, kExpC3 = 0.0552226231f;

__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x2) {
  float x0, x1;
  unpack_f2(x2, x0, x1);
  const uint64_t t = add_f2(pack_f2(fmaxf(x0, -126.f), fmaxf(x1, -126.f)), pack_f2(12582912.f, 12582912.f));
  const uint64_t j = add_f2(t, pack_f2(-12582912.f, -12582912.f));
  float t0, t1, j0, j1;
  unpack_f2(t, t0, t1);
  unpack_f2(j, j0, j1);
  const uint64_t f = pack_f2(fmaxf(x0, -126.f) - j0, fmaxf(x1, -126.f) - j1);
  uint64_t p = fma_f2(pack_f2(kExpC3, kExpC3), f, pack_f2(kExpC2, kExpC2));
  p = fma_f2(p, f, pack_f2(kExpC1, kExpC1));
  p = fma_f2(p, f, pack_f2(kExpC0, kExpC0));
  float p0, p1;
  unpack_f2(p, p0, p1);
  p0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  p1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
  return pack_f2(p0, p1);
}

__device__ __forceinline__ void store_bf16x32(void* dst, const float* v) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 w;
    w.x = pack_bf16x2(v[8 * i + 0], v[8 * i + 1]);
    w.y = pack_bf16x2(v[8 * i + 2], v[8 * i + 3]);
    w.z = pack_bf16x2(v[8 * i + 4], v[8 * i + 5]);
    w.w = pack_bf16x2(v[8 * i + 6], v[8 * i + 7]);
    d[i] = w;
  }
}

__device__ __forceinline__ void store_f32x32(void* dst, const float* v) {
  float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int i = 0; i < 8; ++i) d[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}

__device__ __forceinline__ void load_f32x32(const void* src, float* v) {
  const float4* s = reinterpret_cast<const float4*>(src);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 w = s[i];
    v[4 * i] = w.x;
    v[4 * i + 1] = w.y;
    v[4 * i + 2] = w.z;
    v[4 * i + 3] = w.w;
  }
}

// Where a row parks fp32 element c (0 <= c < HD) of its O_loc between the branch switch and the
// epilogue: the first HD/2 elements in the row's O_full slot, the rest in its D slot (each slot holds
// HD bf16 = HD/2 fp32).  The epilogue reads chunk c (32 elements) before storing O_full chunk c,
// whose bytes [64c, 64c + 64) of the O_full slot park elements [16c, 16c + 16), i.e. chunks <= c/2
// that were read already; D is stored only after every chunk was read.
template <int HD>
__device__ __forceinline__ float* parked(uint8_t* full_row, uint8_t* d_row, int c) {
  return c < HD / 2 ? reinterpret_cast<float*>(full_row) + c : reinterpret_cast<float*>(d_row) + (c - HD / 2);
}

// kBias: a segment may carry a per-key additive logit bias (the log group sizes of a merged cache,
// FAST-AR TempCache); the scores then enter the softmax as s * scale * log2e + bias * log2e.
template <int HD, bool kBias>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ AttnMaps maps, const AttnParams p) {
  using C = Cfg<HD>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023) != 0) {  // the swizzled TMA / UMMA layouts need a 1024-byte aligned base
    if (threadIdx.x == 0) atomicOr(p.status, kStatusInternal);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* full = q_full + 1;
  uint64_t* empty = full + C::kSlots;
  uint64_t* s_full = empty + C::kSlots;  // [2]: S of tile A / B is in TMEM
  uint64_t* p_ready = s_full + 2;        // [2]: P of tile A / B is in TMEM (4 warp arrivals)
  uint64_t* o_final = p_ready + 2;       // every MMA of the CTA has completed
  uint64_t* final_bar = o_final + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  volatile int* never = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 8);  // stays 0: drain waits

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int head = blockIdx.y;
  const int q0 = blockIdx.x * (2 * kBM);
  const bool has_b = q0 + kBM < p.n_q;  // tile B holds at least one query row
  const int T1 = p.tiles[0] + p.tiles[1];
  const int T = T1 + p.tiles[2];
  const bool has_hist = p.tiles[2] > 0;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < C::kSlots; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(p_ready + i, 4);  // one arrival per softmax warp of the tile
    }
    mbar_init(o_final, 1);
    mbar_init(final_bar, 1);
    *abort_flag = 0;
    *never = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ TMA producer
    // (test hook ISPA_TEST_ATTN_NO_LOADS: issue nothing, so every consumer's bounded wait runs out)
    if (lane == 0 && !(p.test_flags & ISPA_TEST_ATTN_NO_LOADS)) {
      tma_prefetch_desc(&maps.q);
      mbar_arrive_expect_tx(q_full, (has_b ? 2 : 1) * C::kQBytes);
      for (int x = 0; x < (has_b ? 2 : 1); ++x) {
#pragma unroll
        for (int b = 0; b < C::kBoxes; ++b)
          tma_load_2d(smem + C::kOffQ + x * C::kQBytes + b * C::kBoxBytes, &maps.q, q_full, head * HD + 64 * b,
                      q0 + x * kBM);
      }
      const int n_loads = 2 * T;  // K_0, V_0, K_1, V_1, ...
      int issued = 0;
      for (int n = 0; n < n_loads; ++n) {
        const int s = n % C::kSlots;
        if (n >= C::kSlots && !mbar_wait(empty + s, ((n / C::kSlots) - 1) & 1, abort_flag)) {
          atomicOr(p.status, kStatusTimeout);
          *abort_flag = 1;
          break;
        }
        int seg, key0, valid;
        tile_info(p, n >> 1, seg, key0, valid);
        const CUtensorMap* map = (n & 1) ? &maps.v[seg] : &maps.k[seg];
        mbar_arrive_expect_tx(full + s, C::kSlotBytes);
#pragma unroll
        for (int b = 0; b < C::kBoxes; ++b)
          tma_load_2d(smem + C::kOffKV + s * C::kSlotBytes + b * C::kBoxBytes, map, full + s, head * HD + 64 * b,
                      key0);
        issued = n + 1;
      }
      // Never leave the CTA with bulk copies in flight: wait for the loads that may be outstanding.
      if (*abort_flag) {
        for (int n = issued - 1; n >= 0 && n >= issued - C::kSlots; --n)
          mbar_wait(full + n % C::kSlots, (n / C::kSlots) & 1, never);
        mbar_wait(q_full, 0, never);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0, abort_flag);
      tc_fence_after();
      const uint32_t q_base = smem_u32(smem + C::kOffQ);
      const uint32_t kv_base = smem_u32(smem + C::kOffKV);
      auto wait_load = [&](int n) -> bool {
        if (!mbar_wait(full + n % C::kSlots, (n / C::kSlots) & 1, abort_flag)) return false;
        tc_fence_after();
        return true;
      };
      auto issue_s = [&](int x, int n) {  // S_x = Q_x K^T, K in the slot of load n
        const uint32_t qb = q_base + x * C::kQBytes;
        const uint32_t kb = kv_base + (n % C::kSlots) * C::kSlotBytes;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kBoxBytes + (kk & 3) * 32;
          umma_ss(tmem + x * 128, sw128_desc(qb + off, 16, 1024), sw128_desc(kb + off, 16, 1024), C::kIdescQK,
                  kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int x, int n, bool first) {  // O_x += P_x V, V in the slot of load n
        const uint32_t vb = kv_base + (n % C::kSlots) * C::kSlotBytes;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          umma_ts(tmem + C::kColO + x * HD, tmem + x * 128 + kk * 8,
                  sw128_desc(vb + kk * 16 * 128, C::kBoxBytes, 1024), C::kIdescPV, (!first || kk > 0) ? 1u : 0u);
      };
      // prologue: S_A(0), S_B(0)
      if (ok) ok = wait_load(0);
      if (ok) {
        issue_s(0, 0);
        umma_commit(s_full + 0);
        if (has_b) {
          issue_s(1, 0);
          umma_commit(s_full + 1);
        }
        umma_commit(empty + 0);  // K_0 consumed
      }
      for (int j = 0; ok && j < T; ++j) {
        const int nv = 2 * j + 1, nk = 2 * j + 2;
        const bool more = j + 1 < T;
        if (!wait_load(nv) || !mbar_wait(p_ready + 0, j & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_pv(0, nv, j == 0);
        if (more) {
          if (!wait_load(nk)) {
            ok = false;
            break;
          }
          issue_s(0, nk);
          umma_commit(s_full + 0);  // also tracks PV_A(j): S_A(j+1) complete implies O_A settled
        }
        if (has_b) {
          if (!mbar_wait(p_ready + 1, j & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(1, nv, j == 0);
        }
        umma_commit(empty + nv % C::kSlots);  // V_j consumed
        if (more) {
          if (has_b) {
            issue_s(1, nk);
            umma_commit(s_full + 1);
          }
          umma_commit(empty + nk % C::kSlots);  // K_(j+1) consumed
        }
      }
      if (!ok) {
        atomicOr(p.status, kStatusTimeout);
        *abort_flag = 1;
      }
      // o_final releases the epilogues; final_bar drains every MMA this thread issued before TMEM is
      // released
      umma_commit(o_final);
      umma_commit(final_bar);
      mbar_wait(final_bar, 0, never);
    }
  } else if ((warp >> 2) == 0 || has_b) {
    // ------------------------------------------------------------------ softmax + epilogue
    const int x = warp >> 2;                  // query tile of this warp
    const int quarter = warp & 3;             // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;      // query row within the tile == TMEM lane
    const int grow = q0 + x * kBM + row;
    const bool live = grow < p.n_q;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_addr = tmem + lane_addr + x * 128;
    const uint32_t o_addr = tmem + lane_addr + C::kColO + x * HD;
    const float sl2 = p.scale_log2;
    const long long off = (static_cast<long long>(grow) * p.ld_o + static_cast<long long>(head) * HD) * 2;
    uint8_t* loc_row = reinterpret_cast<uint8_t*>(p.o_loc) + off;
    uint8_t* full_row = reinterpret_cast<uint8_t*>(p.o_full) + off;
    uint8_t* d_row = p.d_out ? reinterpret_cast<uint8_t*>(p.d_out) + off : nullptr;
    float m = -INFINITY, l_loc = 0.f, l_hist = 0.f, lse_loc2 = 0.f;
    bool alive = true;
    uint32_t r[kBN];
    for (int t = 0; t < T; ++t) {
      alive = mbar_wait_warp(s_full + x, t & 1, abort_flag);
      if (!alive) break;
      tc_fence_after();
      if (t == T1) {
        // branch switch: O holds the local branch alone (PV(T1-1) completed before S(T1) did)
        lse_loc2 = m + __log2f(l_loc);
        const float inv = 1.f / l_loc;
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(o_addr + c * 32, o);
          tmem_wait_ld();
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(o[i]) * inv;
          if (live) {
            store_bf16x32(loc_row + c * 64, v);
            if (d_row) store_f32x32(parked<HD>(full_row, d_row, c * 32), v);
          }
        }
      }
      int seg, key0, valid;
      tile_info(p, t, seg, key0, valid);
      const bool full_tile = valid == kBN;
      const float* brow = nullptr;
      if constexpr (kBias) {
        if (p.bias[seg]) brow = p.bias[seg] + static_cast<long long>(head) * p.ld_bias[seg] + key0;
      }
      if (kBias && brow) {
        // biased scores in log2 units, 32 columns at a time: z = s * scale * log2e + bias * log2e
        constexpr float kLog2e = 1.4426950408889634f;
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) {
          tmem_ld32(s_addr + c * 32, r + c * 32);
          float b[32];
          if (full_tile) {
            const float4* b4 = reinterpret_cast<const float4*>(brow + c * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 w = __ldg(b4 + i);
              b[4 * i] = w.x;
              b[4 * i + 1] = w.y;
              b[4 * i + 2] = w.z;
              b[4 * i + 3] = w.w;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) b[i] = c * 32 + i < valid ? __ldg(brow + c * 32 + i) : -INFINITY;
          }
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i)
            r[c * 32 + i] = __float_as_uint(fmaf(__uint_as_float(r[c * 32 + i]), sl2, b[i] * kLog2e));
        }
      } else {
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) tmem_ld32(s_addr + c * 32, r + c * 32);
        tmem_wait_ld();
        if (!full_tile) {
#pragma unroll
          for (int j = 0; j < kBN; ++j)
            if (j >= valid) r[j] = __float_as_uint(-INFINITY);
        }
      }
      // scores now in r: raw (scaled below by sl2) or, for a biased segment, already in log2 units
      const float rs = (kBias && brow) ? 1.f : sl2;
      // row maximum: a tree of 3-input maxima
      float m8[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float* v = reinterpret_cast<const float*>(r + 8 * i);
        m8[i] = max3f(max3f(v[0], v[1], v[2]), max3f(v[3], v[4], v[5]), fmaxf(v[6], v[7]));
      }
      const float mx = rs * max3f(max3f(max3f(m8[0], m8[1], m8[2]), max3f(m8[3], m8[4], m8[5]),
                                         max3f(m8[6], m8[7], m8[8])),
                                   max3f(m8[9], m8[10], m8[11]), max3f(m8[12], m8[13], fmaxf(m8[14], m8[15])));
      float alpha = 1.f;
      bool rescale = false;
      if (t == 0) {
        m = mx;
      } else if (mx > m + kRescaleThreshold) {
        alpha = fast_exp2(m - mx);
        m = mx;
        rescale = true;
      }
      // exponent arguments two at a time (f32x2 FMA); exp2 on the MUFU unit, except the first
      // kPolyCols columns of full tiles (cubic on the FMA pipe); row sum in two packed
      // accumulators; P packed to bf16 pairs and stored 8 TMEM columns at a time
      const uint64_t sl2x2 = pack_f2(rs, rs), negm2 = pack_f2(-m, -m);
      uint64_t acc[2] = {0ull, 0ull};
#pragma unroll
      for (int c = 0; c < kBN / 16; ++c) {
        uint32_t pk[8];
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
          const int jj = c * 16 + j;
          const uint64_t y = fma_f2(pack_f2(__uint_as_float(r[jj]), __uint_as_float(r[jj + 1])), sl2x2, negm2);
          uint64_t pe;
          if (jj < kPolyCols && full_tile) {
            pe = exp2_poly2(y);
          } else {
            float y0, y1;
            unpack_f2(y, y0, y1);
            pe = pack_f2(fast_exp2(y0), fast_exp2(y1));
          }
          acc[(j >> 1) & 1] = add_f2(acc[(j >> 1) & 1], pe);
          float p0, p1;
          unpack_f2(pe, p0, p1);
          pk[j >> 1] = pack_bf16x2(p0, p1);
        }
        tmem_st8(s_addr + c * 8, pk);
      }
      float a0, a1, a2, a3;
      unpack_f2(acc[0], a0, a1);
      unpack_f2(acc[1], a2, a3);
      const float tile_sum = (a0 + a1) + (a2 + a3);
      l_loc *= alpha;
      l_hist *= alpha;
      if (t < T1)
        l_loc += tile_sum;
      else
        l_hist += tile_sum;
      // tcgen05.ld/st are warp-collective: the warp rescales together if any of its rows needs it
      // (alpha == 1 on the rows that do not).  O is settled here: S(t) completing implies PV(t-1)
      // completed, and PV(t) waits for this warp's p_ready.
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(o_addr + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
          tmem_st32(o_addr + c * 32, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_ready + x);  // one arrival per warp, after the whole warp's stores
    }
    if (alive) alive = mbar_wait_warp(o_final, 0, abort_flag);
    if (!alive) {
      atomicOr(p.status, kStatusTimeout);
      *abort_flag = 1;
    } else {
      tc_fence_after();
      const float ln2 = 0.69314718055994531f;
      if (!has_hist) {
        // no history: O_full is O_loc (the same bf16 values) and D is zero
        const float inv = 1.f / l_loc;
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(o_addr + c * 32, o);
          tmem_wait_ld();
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(o[i]) * inv;
          if (live) {
            store_bf16x32(loc_row + c * 64, v);
            store_bf16x32(full_row + c * 64, v);
            if (d_row) {
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = 0.f;
              store_bf16x32(d_row + c * 64, v);
            }
          }
        }
        if (live) {
          p.lse_loc[(long long)head * p.n_q + grow] = (m + __log2f(l_loc)) * ln2;
          p.lse_hist[(long long)head * p.n_q + grow] = -INFINITY;
        }
      } else {
        const float inv = 1.f / (l_loc + l_hist);
        uint32_t dpk[HD / 2];  // D, packed, stored once every parked chunk has been read
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(o_addr + c * 32, o);
          tmem_wait_ld();
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(o[i]) * inv;
          if (live) {
            if (d_row) {
              float ol[32];
              load_f32x32(parked<HD>(full_row, d_row, c * 32), ol);
#pragma unroll
              for (int i = 0; i < 32; i += 2) dpk[c * 16 + i / 2] = pack_bf16x2(v[i] - ol[i], v[i + 1] - ol[i + 1]);
            }
            store_bf16x32(full_row + c * 64, v);
          }
        }
        if (live && d_row) {
          uint4* dst = reinterpret_cast<uint4*>(d_row);
#pragma unroll
          for (int i = 0; i < HD / 8; ++i) dst[i] = make_uint4(dpk[4 * i], dpk[4 * i + 1], dpk[4 * i + 2], dpk[4 * i + 3]);
        }
        if (live) {
          p.lse_loc[(long long)head * p.n_q + grow] = lse_loc2 * ln2;
          p.lse_hist[(long long)head * p.n_q + grow] = (m + __log2f(l_hist)) * ln2;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool attn_tc_supported(const AttnLaunch& a) {
  if (a.dtype != 0) return false;
  if (a.head_dim != 64 && a.head_dim != 128) return false;
  if (a.n_q > (1ll << 30)) return false;
  auto al16 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; };
  if (!al16(a.q) || (a.ld_q % 8) != 0) return false;
  for (int s = 0; s < 3; ++s) {
    if (a.n_kv[s] == 0) continue;
    if (a.n_kv[s] > (1ll << 30)) return false;
    if (!al16(a.k[s]) || !al16(a.v[s]) || (a.ld_k[s] % 8) || (a.ld_v[s] % 8)) return false;
  }
  if (!al16(a.o_loc) || !al16(a.o_full) || (a.d_out && !al16(a.d_out)) || (a.ld_o % 8)) return false;
  for (int s = 0; s < 3; ++s)  // vector loads of a full tile's 128 biases
    if (a.bias[s] && a.n_kv[s] > 0 && (!al16(a.bias[s]) || (a.ld_bias[s] % 4))) return false;
  return true;
}

template <int HD, bool kBias>
static cudaError_t launch_hd(const AttnLaunch& a, cudaStream_t stream, int* n_launched) {
  using C = Cfg<HD>;
  AttnMaps maps;
  memset(&maps, 0, sizeof(maps));
  const uint64_t d = static_cast<uint64_t>(a.n_heads) * HD;
  if (!make_map_bf16_2d(&maps.q, a.q, a.n_q, d, a.ld_q, 64, kBM)) return cudaErrorInvalidValue;
  AttnParams p;
  memset(&p, 0, sizeof(p));
  for (int s = 0; s < 3; ++s) {
    p.n_kv[s] = static_cast<int>(a.n_kv[s]);
    p.tiles[s] = static_cast<int>((a.n_kv[s] + kBN - 1) / kBN);
    if (a.n_kv[s] > 0) {
      if (!make_map_bf16_2d(&maps.k[s], a.k[s], a.n_kv[s], d, a.ld_k[s], 64, kBN)) return cudaErrorInvalidValue;
      if (!make_map_bf16_2d(&maps.v[s], a.v[s], a.n_kv[s], d, a.ld_v[s], 64, kBN)) return cudaErrorInvalidValue;
    }
  }
  p.n_q = static_cast<int>(a.n_q);
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.o_loc = a.o_loc;
  p.o_full = a.o_full;
  p.d_out = a.d_out;
  p.ld_o = a.ld_o;
  p.lse_loc = a.lse_loc;
  p.lse_hist = a.lse_hist;
  p.status = a.status;
  p.test_flags = a.test_flags;
  for (int s = 0; s < 3; ++s) {
    p.bias[s] = a.n_kv[s] > 0 ? a.bias[s] : nullptr;
    p.ld_bias[s] = a.ld_bias[s];
  }
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<HD, kBias>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>((a.n_q + 2 * kBM - 1) / (2 * kBM)), static_cast<unsigned>(a.n_heads));
  attn_tc_kernel<HD, kBias><<<grid, kThreads, C::kSmemBytes, stream>>>(maps, p);
  *n_launched += 1;
  return cudaGetLastError();
}

cudaError_t launch_attn_tc(const AttnLaunch& a, cudaStream_t s, int* n_launched) {
  if (a.n_q == 0) return cudaSuccess;
  const bool biased = a.bias[0] || a.bias[1] || a.bias[2];
  if (a.head_dim == 128) return biased ? launch_hd<128, true>(a, s, n_launched) : launch_hd<128, false>(a, s, n_launched);
  return biased ? launch_hd<64, true>(a, s, n_launched) : launch_hd<64, false>(a, s, n_launched);
}

}  // namespace ispa
