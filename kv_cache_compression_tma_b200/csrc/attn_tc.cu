// attn_tc.cu -- decomposable (dual-stream) attention on tcgen05 tensor cores, sm_100a.
//
// ISPA summary, section 2, stage 1 ("Decomposable Attention"): one pass over the KV cache yields
// both A_loc (sink + current chunk) and A_full (sink + current chunk + history) by keeping the
// online-softmax state of the two key branches apart and merging them post-hoc by log-sum-exp.
//
// One CTA computes one (128-query-row tile, head).  Keys are walked once, in the order
// sink tiles, local tiles (the local branch), history tiles (the history branch).  Each branch owns
// its running max m, running sum l and fp32 accumulator in TMEM, so at the end
//   O_loc  = O_A / l_loc,   O_hist = O_B / l_hist,
//   O_full = w_loc O_loc + w_hist O_hist with w = softmax over (lse_loc, lse_hist),
//   D      = O_full - O_loc  (formed in fp32 before rounding).
//
// Warp roles (320 threads):
//   warp 0      TMA producer: Q once, then K and V tiles of 128 keys into a ring of NST stages
//   warp 1      TMEM owner + single-thread MMA issuer:
//                 S_t = Q K_t^T          (SS MMA, bf16 -> fp32, into TMEM S buffer t%2)
//                 O_branch += P_t V_t    (TS MMA: P read from TMEM, V from shared memory)
//   warps 2..9  softmax + epilogue, two threads per query row r (TMEM lane r): warps 2..5 own key
//               columns 0..63 of S_t, warps 6..9 columns 64..127.  The pair exchanges its partial row
//               max through shared memory (one 64-thread named barrier per row quarter), writes
//               P_t = exp2(S_t*scale*log2e - m) as bf16 into the same TMEM columns, keeps a partial
//               row sum, and rescales its half of the branch accumulator only when the row max grows
//               by more than 2^8.
// TMEM columns: [0,128) S/P buffer 0, [128,256) S/P buffer 1, [256,256+HD) O_A, then O_B.
// Every barrier wait is bounded (see sm100.cuh); a timeout records ISPA_ERR_TIMEOUT and unwinds.
#include <math.h>
#include <string.h>

#include "../../include/ispa.h"
#include "internal.h"
#include "sm100.cuh"

namespace ispa {
namespace {

constexpr int kBM = 128;   // query rows per CTA
constexpr int kBN = 128;   // keys per tile
constexpr int kThreads = 320;
constexpr int kSoftmaxThreads = 256;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

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
  static constexpr int kBoxes = HD / 64;                  // 128-byte boxes per row
  static constexpr int kBoxBytesQ = kBM * 128;            // one 64-column box of 128 rows
  static constexpr int kBoxBytesKV = kBN * 128;
  static constexpr int kQBytes = kBM * HD * 2;
  static constexpr int kTileBytes = kBN * HD * 2;
  static constexpr int kStages = (HD == 128) ? 3 : 4;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kStages * kTileBytes;
  // barriers: q_full, k_full[S], v_full[S], kv_empty[S], s_full[2], p_ready[2], o_done, o_final, final
  static constexpr int kNumBars = 1 + 3 * kStages + 2 + 2 + 1 + 1 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffXchg = kOffMisc + 16;                    // [2 tiles][2 halves][128 rows] float
  static constexpr int kSmemBytes = kOffXchg + 2 * 2 * kBM * 4;    // base is 1024-byte aligned
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, kBN, false, false);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, HD, false, true);
  static_assert(kSmemBytes <= 232448, "shared memory budget");
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

// kBias: a segment may carry a per-key additive logit bias (the log group sizes of a merged cache,
// FAST-AR TempCache); its scores then enter the softmax as s * scale * log2e + bias * log2e.
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
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + C::kStages;
  uint64_t* kv_empty = v_full + C::kStages;
  uint64_t* s_full = kv_empty + C::kStages;
  uint64_t* p_ready = s_full + 2;
  uint64_t* o_done = p_ready + 2;
  uint64_t* o_final = o_done + 1;  // once: every MMA of the CTA has completed
  uint64_t* final_bar = o_final + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  volatile int* never = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 8);  // stays 0: drain waits

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int head = blockIdx.y;
  const int q0 = blockIdx.x * kBM;
  const int T1 = p.tiles[0] + p.tiles[1];
  const int T = T1 + p.tiles[2];

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(v_full + i, 1);
      mbar_init(kv_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(p_ready + i, kSoftmaxThreads / 32);  // one arrival per softmax warp
    }
    mbar_init(o_done, 1);
    mbar_init(o_final, 1);
    mbar_init(final_bar, 1);
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
    // ------------------------------------------------------------------ TMA producer
    // (test hook ISPA_TEST_ATTN_NO_LOADS: issue nothing, so every consumer's bounded wait runs out)
    if (lane == 0 && !(p.test_flags & ISPA_TEST_ATTN_NO_LOADS)) {
      tma_prefetch_desc(&maps.q);
      mbar_arrive_expect_tx(q_full, C::kQBytes);
#pragma unroll
      for (int b = 0; b < C::kBoxes; ++b)
        tma_load_2d(smem + C::kOffQ + b * C::kBoxBytesQ, &maps.q, q_full, head * HD + 64 * b, q0);
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const int s = t % C::kStages;
        if (t >= C::kStages) {
          if (!mbar_wait(kv_empty + s, ((t / C::kStages) - 1) & 1, abort_flag)) {
            atomicOr(p.status, kStatusTimeout);
            *abort_flag = 1;
            break;
          }
        }
        int seg, key0, valid;
        tile_info(p, t, seg, key0, valid);
        mbar_arrive_expect_tx(k_full + s, C::kTileBytes);
#pragma unroll
        for (int b = 0; b < C::kBoxes; ++b)
          tma_load_2d(smem + C::kOffK + s * C::kTileBytes + b * C::kBoxBytesKV, &maps.k[seg], k_full + s,
                      head * HD + 64 * b, key0);
        mbar_arrive_expect_tx(v_full + s, C::kTileBytes);
#pragma unroll
        for (int b = 0; b < C::kBoxes; ++b)
          tma_load_2d(smem + C::kOffV + s * C::kTileBytes + b * C::kBoxBytesKV, &maps.v[seg], v_full + s,
                      head * HD + 64 * b, key0);
        issued = t + 1;
      }
      // Never leave the CTA with bulk copies in flight: wait for the last load of every stage.
      if (*abort_flag) {
        for (int t = issued - 1; t >= 0 && t >= issued - C::kStages; --t) {
          const int s = t % C::kStages;
          mbar_wait(k_full + s, (t / C::kStages) & 1, never);
          mbar_wait(v_full + s, (t / C::kStages) & 1, never);
        }
        mbar_wait(q_full, 0, never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0, abort_flag);
      tc_fence_after();
      const uint32_t q_base = smem_u32(smem + C::kOffQ);
      auto issue_pv = [&](int u) -> bool {
        const int b = u & 1;
        const int s = u % C::kStages;
        if (!mbar_wait(p_ready + b, (u >> 1) & 1, abort_flag)) return false;
        if (!mbar_wait(v_full + s, (u / C::kStages) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t o_tmem = tmem + 256 + (u >= T1 ? HD : 0);
        const bool first = (u == 0) || (u == T1);
        const uint32_t v_base = smem_u32(smem + C::kOffV + s * C::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t bdesc = sw128_desc(v_base + kk * 16 * 128, C::kBoxBytesKV, 1024);
          umma_ts(o_tmem, tmem + b * 128 + kk * 8, bdesc, C::kIdescPV, (!first || kk > 0) ? 1u : 0u);
        }
        umma_commit(o_done);
        umma_commit(kv_empty + s);
        return true;
      };
      for (int t = 0; ok && t < T; ++t) {
        const int s = t % C::kStages;
        if (!mbar_wait(k_full + s, (t / C::kStages) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_base = smem_u32(smem + C::kOffK + s * C::kTileBytes);
        const uint32_t d_tmem = tmem + (t & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kBoxBytesQ + (kk & 3) * 32;
          const uint64_t adesc = sw128_desc(q_base + off, 16, 1024);
          const uint64_t bdesc = sw128_desc(k_base + (kk >> 2) * C::kBoxBytesKV + (kk & 3) * 32, 16, 1024);
          umma_ss(d_tmem, adesc, bdesc, C::kIdescQK, kk > 0 ? 1u : 0u);
        }
        umma_commit(s_full + (t & 1));
        if (t > 0 && !issue_pv(t - 1)) {
          ok = false;
          break;
        }
      }
      if (ok && T > 0) ok = issue_pv(T - 1);
      if (!ok) {
        atomicOr(p.status, kStatusTimeout);
        *abort_flag = 1;
      }
      // o_final releases the epilogue; final_bar drains every MMA this thread issued before TMEM is
      // released
      umma_commit(o_final);
      umma_commit(final_bar);
      mbar_wait(final_bar, 0, never);
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int quarter = warp & 3;             // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;         // which 64 key columns of S (and HD/2 columns of O)
    const int row = quarter * 32 + lane;      // query row within the tile == TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    float* xchg = reinterpret_cast<float*>(smem + C::kOffXchg);  // [tile parity][half][row]
    const int bar_id = 1 + quarter;           // named barrier of this row quarter's two warps
    const float sl2 = p.scale_log2;
    constexpr int kCols = kBN / 2;            // S columns per thread
    constexpr int kOCols = HD / 2;            // O columns per thread
    float m = -INFINITY, l = 0.f;             // l: partial row sum over this thread's columns
    float m_loc = -INFINITY, l_loc = 0.f;
    // `alive` is warp-uniform.  A warp whose bounded wait ran out stops working but keeps executing
    // one pair barrier per tile, so the two warps of a row quarter always meet the same number of
    // times (no early exit from the loop).
    bool alive = true;
    uint32_t r[kCols];
    for (int t = 0; t < T; ++t) {
      const int b = t & 1;
      int seg, key0, valid;
      tile_info(p, t, seg, key0, valid);
      if (t == T1) {  // branch switch: freeze the local branch, start the history branch
        m_loc = m;
        l_loc = l;
        m = -INFINITY;
        l = 0.f;
      }
      const bool first = (t == 0) || (t == T1);
      if (alive) alive = mbar_wait_warp(s_full + b, (t >> 1) & 1, abort_flag);
      const uint32_t s_addr = tmem + lane_addr + b * 128;
      float mx = -INFINITY;
      const int lim = valid - half * kCols;  // columns of this half that hold real keys
      // scores in r are raw (scaled by sl2 below) or, on a biased segment, already in log2 units
      float rs = sl2;
      if (alive) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < kCols / 32; ++c) tmem_ld32(s_addr + half * kCols + c * 32, r + c * 32);
        const float* brow = nullptr;
        if constexpr (kBias) {
          if (p.bias[seg]) brow = p.bias[seg] + static_cast<long long>(head) * p.ld_bias[seg] + key0 + half * kCols;
        }
        if (kBias && brow) {
          constexpr float kLog2e = 1.4426950408889634f;
          float bb[kCols];
          if (lim >= kCols) {
            const float4* b4 = reinterpret_cast<const float4*>(brow);
#pragma unroll
            for (int i = 0; i < kCols / 4; ++i) {
              const float4 w = __ldg(b4 + i);
              bb[4 * i] = w.x;
              bb[4 * i + 1] = w.y;
              bb[4 * i + 2] = w.z;
              bb[4 * i + 3] = w.w;
            }
          } else {
#pragma unroll
            for (int j = 0; j < kCols; ++j) bb[j] = j < lim ? __ldg(brow + j) : -INFINITY;
          }
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < kCols; ++j) r[j] = __float_as_uint(fmaf(__uint_as_float(r[j]), sl2, bb[j] * kLog2e));
          rs = 1.f;
        } else {
          tmem_wait_ld();
        }
        if (lim >= kCols) {
          // tree of 3-input maxima: 8 independent partial maxima of 8 columns, then 3 more levels
          float m8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float* v = reinterpret_cast<const float*>(r + 8 * i);
            m8[i] = max3f(max3f(v[0], v[1], v[2]), max3f(v[3], v[4], v[5]), fmaxf(v[6], v[7]));
          }
          mx = max3f(max3f(m8[0], m8[1], m8[2]), max3f(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
        } else {
#pragma unroll
          for (int j = 0; j < kCols; ++j) {
            const float x = j < lim ? __uint_as_float(r[j]) : -INFINITY;
            r[j] = __float_as_uint(x);
            mx = fmaxf(mx, x);
          }
        }
      }
      // row max over both halves
      xchg[(b * 2 + half) * kBM + row] = mx;
      asm volatile("bar.sync %0, 64;" ::"r"(bar_id) : "memory");
      mx = fmaxf(xchg[(b * 2) * kBM + row], xchg[(b * 2 + 1) * kBM + row]) * rs;
      if (!alive) continue;
      bool rescale = false;
      float alpha = 1.f;
      if (first) {
        m = mx;
      } else if (mx > m + kRescaleThreshold) {
        alpha = fast_exp2(m - mx);
        m = mx;
        rescale = true;
      }
      // exponent arguments two at a time (f32x2 FMA), exp2 on the XU pipe, row sum in four packed
      // accumulators (f32x2 adds), P packed to bf16 pairs
      const uint64_t sl2x2 = pack_f2(rs, rs), negm2 = pack_f2(-m, -m);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
      uint32_t pk[kCols / 2];
#pragma unroll
      for (int j = 0; j < kCols; j += 2) {
        const uint64_t y = fma_f2(pack_f2(__uint_as_float(r[j]), __uint_as_float(r[j + 1])), sl2x2, negm2);
        float y0, y1;
        unpack_f2(y, y0, y1);
        const float p0 = fast_exp2(y0), p1 = fast_exp2(y1);
        acc[(j >> 1) & 3] = add_f2(acc[(j >> 1) & 3], pack_f2(p0, p1));
        pk[j >> 1] = pack_bf16x2(p0, p1);
      }
      float a0, a1, a2, a3, a4, a5, a6, a7;
      unpack_f2(acc[0], a0, a1);
      unpack_f2(acc[1], a2, a3);
      unpack_f2(acc[2], a4, a5);
      unpack_f2(acc[3], a6, a7);
      l = l * alpha + (((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7)));
      tmem_st32(s_addr + half * (kCols / 2), pk);
      // tcgen05.ld/st are warp-collective: the warp rescales together if any of its rows needs it
      // (alpha == 1 on the rows that do not).  Only then must PV_{t-1} be complete; P_t goes to the
      // MMA without waiting for it (the tensor core runs PV_{t-1} before PV_t).  S_t complete
      // implies PV_{t-2} complete, and PV_t needs this warp's p_ready, so o_done has completed
      // t-1 or t phases here and the parity wait for phase t-1 cannot alias.
      if (__any_sync(0xffffffffu, rescale)) {
        if (t > 0) alive = mbar_wait_warp(o_done, (t - 1) & 1, abort_flag);
      }
      if (!alive) continue;
      if (__any_sync(0xffffffffu, rescale)) {
        tc_fence_after();
        const uint32_t o_addr = tmem + lane_addr + 256 + (t >= T1 ? HD : 0) + half * kOCols;
#pragma unroll
        for (int c = 0; c < kOCols / 32; ++c) {
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
      if (lane == 0) mbar_arrive(p_ready + b);  // one arrival per warp, after the whole warp's stores
    }
    if (alive && T > 0) alive = mbar_wait_warp(o_final, 0, abort_flag);
    const bool ok = alive;
    // partial row sums of the two halves (the exchange buffer is free: every pair passed its last
    // max exchange before its last p_ready, which the last PV, and so o_final, waited for)
    const bool has_hist = p.tiles[2] > 0;
    if (!has_hist) {
      m_loc = m;
      l_loc = l;
    }
    xchg[half * kBM + row] = l_loc;
    xchg[(2 + half) * kBM + row] = l;
    asm volatile("bar.sync %0, 64;" ::"r"(bar_id) : "memory");
    const float l_loc_row = xchg[row] + xchg[kBM + row];
    const float l_hist_row = xchg[2 * kBM + row] + xchg[3 * kBM + row];
    if (!ok) {
      atomicOr(p.status, kStatusTimeout);
      *abort_flag = 1;
    } else {
      tc_fence_after();
      const float lse_loc2 = m_loc + __log2f(l_loc_row);
      const float lse_hist2 = has_hist ? m + __log2f(l_hist_row) : -INFINITY;
      float w_loc = 1.f, w_hist = 0.f;
      if (has_hist) {
        const float mm = fmaxf(lse_loc2, lse_hist2);
        const float a = exp2f(lse_loc2 - mm), bb = exp2f(lse_hist2 - mm);
        w_loc = a / (a + bb);
        w_hist = bb / (a + bb);
      }
      const float inv_l_loc = 1.f / l_loc_row;
      const float inv_l_hist = has_hist ? 1.f / l_hist_row : 0.f;
      const int grow = q0 + row;
      const bool live = grow < p.n_q;
      const uint32_t oa_addr = tmem + lane_addr + 256 + half * kOCols;
      const uint32_t ob_addr = oa_addr + HD;
      const long long col0 = static_cast<long long>(head) * HD + half * kOCols;
      __nv_bfloat16* o_loc_row = reinterpret_cast<__nv_bfloat16*>(p.o_loc) + (long long)grow * p.ld_o + col0;
      __nv_bfloat16* o_full_row = reinterpret_cast<__nv_bfloat16*>(p.o_full) + (long long)grow * p.ld_o + col0;
      __nv_bfloat16* d_row =
          p.d_out ? reinterpret_cast<__nv_bfloat16*>(p.d_out) + (long long)grow * p.ld_o + col0 : nullptr;
#pragma unroll 1
      for (int c = 0; c < kOCols / 32; ++c) {
        uint32_t oa[32], ob[32];
        tmem_ld32(oa_addr + c * 32, oa);
        if (has_hist) tmem_ld32(ob_addr + c * 32, ob);
        tmem_wait_ld();
        float vl[32], vf[32], vd[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          vl[j] = __uint_as_float(oa[j]) * inv_l_loc;
          vf[j] = has_hist ? fmaf(w_loc, vl[j], w_hist * (__uint_as_float(ob[j]) * inv_l_hist)) : vl[j];
          vd[j] = vf[j] - vl[j];
        }
        if (live) {
          store_bf16x32(o_loc_row + c * 32, vl);
          store_bf16x32(o_full_row + c * 32, vf);
          if (d_row) store_bf16x32(d_row + c * 32, vd);
        }
      }
      if (live && half == 0) {
        const float ln2 = 0.69314718055994531f;
        p.lse_loc[(long long)head * p.n_q + grow] = lse_loc2 * ln2;
        p.lse_hist[(long long)head * p.n_q + grow] = has_hist ? lse_hist2 * ln2 : -INFINITY;
      }
    }
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
  for (int s = 0; s < 3; ++s)  // vector loads of a half tile's 64 biases
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
  dim3 grid(static_cast<unsigned>((a.n_q + kBM - 1) / kBM), static_cast<unsigned>(a.n_heads));
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
