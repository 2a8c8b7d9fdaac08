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
// Warp roles (96 + 128 * kSplit threads; kSplit = 2 softmax threads per query row, 4 when the call
// carries a per-key bias):
//   warp 0      TMA producer of Q (once) and of the two-stage K ring
//   warp 2      TMA producer of the two-stage V ring (with the tile's bias row, when there is one)
//   warp 1      TMEM owner + single-thread MMA issuer:
//                 S_t = Q K_t^T          (SS MMA, bf16 -> fp32, into TMEM S buffer t%2)
//                 O_branch += P_t V_t    (TS MMA: P read from TMEM, V from shared memory)
//               Two tcgen05.commit per tile: s_full[t%2] (S_t ready, K_t's stage free) and
//               o_done[t%2] (O += P_t V_t done, V_t's stage free).
//   warps 3..   softmax + epilogue, kSplit threads per query row r (TMEM lane r), each on 128/kSplit
//               key columns of S_t.  The row's parts combine their maxima by a shared-memory atomic
//               max (one named barrier per row quarter), write P_t = exp2(S_t*scale*log2e - m) as bf16
//               into the same TMEM columns, keep partial row sums, and rescale their columns of the
//               branch accumulator only when the row max grows by more than 2^8.  The epilogue
//               stages O_loc, O_full and D in the then idle K/V rings (128-byte swizzle) and one
//               thread writes them with bulk tensor stores.
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
constexpr int kFirstSoftmaxWarp = 3;  // warps 0..2: K producer, MMA issuer, V producer
// threads of a CTA with kSplit softmax threads per query row (2, or 4 where a per-key bias adds
// registers to the softmax)
constexpr int threads_for(int split) { return 32 * kFirstSoftmaxWarp + 128 * split; }
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct AttnMaps {
  CUtensorMap q;
  CUtensorMap k[3];
  CUtensorMap v[3];
  CUtensorMap out[3];  // O_loc, O_full, D: {64 cols, 128 rows} boxes for the epilogue's bulk stores
};

struct AttnParams {
  int n_q;
  int n_kv[3];
  int tiles[3];
  float scale_log2;
  void* o_loc;  // the outputs leave through the tensor maps; the pointers are kept for reference
  void* o_full;
  void* d_out;  // null: no D output
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
  // Two-stage K and V rings, one stage per S/P buffer: K_t is released by the same MMA completion that
  // publishes S_t (s_full), V_t and the tile's bias row by the one that publishes O += P_t V_t
  // (o_done), so each tile costs two tcgen05.commit, not four.
  static constexpr int kKStages = 2;
  static constexpr int kVStages = 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kKStages * kTileBytes;
  static constexpr int kOffBias = kOffV + kVStages * kTileBytes;  // [kVStages][kBN] float
  static constexpr int kOffBar = kOffBias + kVStages * kBN * 4;
  // barriers: q_full, k_full[2], v_full[2], s_full[2], p_ready[2], o_done[2], o_final, final
  static constexpr int kNumBars = 1 + kKStages + kVStages + 2 + 2 + 2 + 1 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffXchg = kOffMisc + 16;                    // [3 slots][128 rows] row maxima
  static constexpr int kSmemBytes = kOffXchg + 3 * kBM * 4;         // base is 1024-byte aligned
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

// 2-D tiled bulk tensor store shared -> global (bulk-group completion); rows past the tensor's end are
// not written.
__device__ __forceinline__ void store_tile_2d(const CUtensorMap* map, const void* smem_src, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(smem_src)), "r"(x), "r"(y)
               : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem_attn() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Staging tile of output w (0 O_loc, 1 O_full, 2 D) in the K/V rings, free once every MMA is done.
template <int HD>
__device__ __forceinline__ uint8_t* stage_out_base(uint8_t* smem, int w) {
  using C = Cfg<HD>;
  return w == 0 ? smem + C::kOffV : (w == 1 ? smem + C::kOffV + C::kTileBytes : smem + C::kOffK + C::kTileBytes);
}

__device__ __forceinline__ float4 lds_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}

// N consecutive 32-bit TMEM columns of this thread's lane (N = 16 or 32).
template <int N>
__device__ __forceinline__ void tmem_ld_n(uint32_t taddr, uint32_t* r) {
  if constexpr (N == 32)
    tmem_ld32(taddr, r);
  else
    tmem_ld16(taddr, r);
}
template <int N>
__device__ __forceinline__ void tmem_st_n(uint32_t taddr, const uint32_t* r) {
  if constexpr (N == 32)
    tmem_st32(taddr, r);
  else
    tmem_st16(taddr, r);
}

// kBias: a segment may carry a per-key additive logit bias (the log group sizes of a merged cache,
// FAST-AR TempCache): its exponent arguments are s * scale * log2e + (bias * log2e - m), one more
// packed FMA per pair, while the running maximum m stays over the unbiased scores (a bias of at
// most 16 raises P by at most e^16, well inside fp32 and bf16 range).
template <int HD, bool kBias, int kSplit>
__global__ void __launch_bounds__(threads_for(kSplit), 1)
    attn_tc_kernel(const __grid_constant__ AttnMaps maps, const AttnParams p) {
  using C = Cfg<HD>;
  static_assert(kSplit == 2 || kSplit == 4, "two or four softmax threads per query row");
  constexpr int kSoftmaxThreads = 128 * kSplit;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023) != 0) {  // the swizzled TMA / UMMA layouts need a 1024-byte aligned base
    if (threadIdx.x == 0) atomicOr(p.status, kStatusInternal);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + C::kKStages;
  uint64_t* s_full = v_full + C::kVStages;  // s_full[b]: S_t complete (K_t free), tiles t % 2 == b
  uint64_t* p_ready = s_full + 2;
  uint64_t* o_done = p_ready + 2;           // o_done[b]: O += P_t V_t complete (V_t free), t % 2 == b
  uint64_t* o_final = o_done + 2;           // once: every MMA of the CTA has completed
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
    for (int i = 0; i < 2; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(v_full + i, 1);
      mbar_init(s_full + i, 1);
      mbar_init(p_ready + i, kSoftmaxThreads / 32);  // one arrival per softmax warp
      mbar_init(o_done + i, 1);
    }
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

  if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------------ TMA producers
    // warp 0: Q once, then the K ring; warp 2: the V ring, with the tile's bias row when the segment
    // has one and the tile is full (a partial tile's biases are read from global memory by the
    // softmax).  (Test hook ISPA_TEST_ATTN_NO_LOADS: issue nothing, so every consumer's bounded wait
    // runs out.)
    if (lane == 0 && !(p.test_flags & ISPA_TEST_ATTN_NO_LOADS)) {
      const bool is_k = warp == 0;
      const int n_st = is_k ? C::kKStages : C::kVStages;
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? s_full : o_done;  // stage t % 2 frees with the MMA of tile t - 2
      if (is_k) {
        tma_prefetch_desc(&maps.q);
        mbar_arrive_expect_tx(q_full, C::kQBytes);
#pragma unroll
        for (int b = 0; b < C::kBoxes; ++b)
          tma_load_2d(smem + C::kOffQ + b * C::kBoxBytesQ, &maps.q, q_full, head * HD + 64 * b, q0);
      }
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const int s = t % n_st;
        if (t >= n_st && !mbar_wait(empty + s, ((t / n_st) - 1) & 1, abort_flag)) {
          atomicOr(p.status, kStatusTimeout);
          *abort_flag = 1;
          break;
        }
        int seg, key0, valid;
        tile_info(p, t, seg, key0, valid);
        const float* brow = nullptr;  // 512 bytes from a 16-byte aligned row (checked on the host)
        if constexpr (kBias) {
          if (!is_k && p.bias[seg] && valid == kBN)
            brow = p.bias[seg] + static_cast<long long>(head) * p.ld_bias[seg] + key0;
        }
        mbar_arrive_expect_tx(full + s, C::kTileBytes + (brow ? kBN * 4 : 0));
        const CUtensorMap* map = is_k ? &maps.k[seg] : &maps.v[seg];
        uint8_t* dst = smem + (is_k ? C::kOffK : C::kOffV) + s * C::kTileBytes;
#pragma unroll
        for (int b = 0; b < C::kBoxes; ++b) tma_load_2d(dst + b * C::kBoxBytesKV, map, full + s, head * HD + 64 * b, key0);
        if (brow) bulk_load(smem + C::kOffBias + s * kBN * 4, brow, kBN * 4, full + s);
        issued = t + 1;
      }
      // Never leave the CTA with bulk copies in flight: wait for the last load of every stage.
      if (*abort_flag) {
        for (int t = issued - 1; t >= 0 && t >= issued - n_st; --t) mbar_wait(full + (t % n_st), (t / n_st) & 1, never);
        if (is_k) mbar_wait(q_full, 0, never);
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
        const int s = u % C::kVStages;
        if (!mbar_wait(p_ready + b, (u >> 1) & 1, abort_flag)) return false;
        if (!mbar_wait(v_full + s, (u / C::kVStages) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t o_tmem = tmem + 256 + (u >= T1 ? HD : 0);
        const bool first = (u == 0) || (u == T1);
        const uint32_t v_base = smem_u32(smem + C::kOffV + s * C::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t bdesc = sw128_desc(v_base + kk * 16 * 128, C::kBoxBytesKV, 1024);
          umma_ts(o_tmem, tmem + b * 128 + kk * 8, bdesc, C::kIdescPV, (!first || kk > 0) ? 1u : 0u);
        }
        umma_commit(o_done + b);  // also frees V_u's stage (u % 2 == b)
        return true;
      };
      for (int t = 0; ok && t < T; ++t) {
        const int s = t % C::kKStages;
        if (!mbar_wait(k_full + s, (t / C::kKStages) & 1, abort_flag)) {
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
        umma_commit(s_full + (t & 1));  // also frees K_t's stage (t % 2)
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
    const int part = (warp - kFirstSoftmaxWarp) >> 2;  // which kBN/kSplit key columns of S (HD/kSplit of O)
    const int row = quarter * 32 + lane;      // query row within the tile == TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    // Row maxima of the key tiles: slot t % 3 collects tile t's maximum over the row's parts by a
    // shared-memory atomic max on order-preserving integer images of the floats; part 0 clears the
    // slot of tile t-1 after the barrier of tile t (every part has read it by then), ready for t+2.
    int* mslot = reinterpret_cast<int*>(smem + C::kOffXchg);
    auto ordered = [](int i) { return i >= 0 ? i : i ^ 0x7fffffff; };  // an involution
    const int kNegInf = ordered(__float_as_int(-INFINITY));
    const int bar_id = 1 + quarter;           // named barrier of this row quarter's kSplit warps
    constexpr int kBarThreads = 32 * kSplit;
    const float sl2 = p.scale_log2;
    constexpr int kCols = kBN / kSplit;       // S columns per thread
    constexpr int kOCols = HD / kSplit;       // O columns per thread
    constexpr int kOC = kOCols < 32 ? kOCols : 32;             // O columns per TMEM access (rescale)
    constexpr int kEC = (kSplit == 4 && kOCols >= 16) ? 16 : kOC;  // per epilogue step (registers)
    float m = -INFINITY, l = 0.f;             // l: partial row sum over this thread's columns
    float m_loc = -INFINITY, l_loc = 0.f;
    // `alive` is warp-uniform.  A warp whose bounded wait ran out stops working but keeps executing
    // one pair barrier per tile, so the two warps of a row quarter always meet the same number of
    // times (no early exit from the loop).
    bool alive = true;
    if (part == 0)
#pragma unroll
      for (int i = 0; i < 3; ++i) mslot[i * kBM + row] = kNegInf;
    asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "n"(kBarThreads) : "memory");
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
      const int lim = valid - part * kCols;  // columns of this part that hold real keys
      // a biased segment adds bias * log2e to each score inside the exponent (below); the row maximum
      // is taken over the raw scores: the bias (the log of a group size) only raises P by that size
      // This part's biases: staged in shared memory with V_t (full tiles), or read from global memory
      // (the partial last tile of a segment).
      const float* brow = nullptr;
      bool bias_smem = false;
      if constexpr (kBias) {
        if (p.bias[seg]) {
          bias_smem = valid == kBN;
          brow = bias_smem ? reinterpret_cast<const float*>(smem + C::kOffBias + (t % C::kVStages) * kBN * 4) + part * kCols
                           : p.bias[seg] + static_cast<long long>(head) * p.ld_bias[seg] + key0 + part * kCols;
        }
      }
      if (alive) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < kCols / 32; ++c) tmem_ld32(s_addr + part * kCols + c * 32, r + c * 32);
        tmem_wait_ld();
        if (lim >= kCols) {
          // tree of 3-input maxima: independent partial maxima of 8 columns, then their maximum
          float m8[kCols / 8];
#pragma unroll
          for (int i = 0; i < kCols / 8; ++i) {
            const float* v = reinterpret_cast<const float*>(r + 8 * i);
            m8[i] = max3f(max3f(v[0], v[1], v[2]), max3f(v[3], v[4], v[5]), fmaxf(v[6], v[7]));
          }
          if constexpr (kCols == 64)
            mx = max3f(max3f(m8[0], m8[1], m8[2]), max3f(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
          else
            mx = fmaxf(max3f(m8[0], m8[1], m8[2]), m8[3]);
        } else {
#pragma unroll
          for (int j = 0; j < kCols; ++j) {
            const float x = j < lim ? __uint_as_float(r[j]) : -INFINITY;
            r[j] = __float_as_uint(x);
            mx = fmaxf(mx, x);
          }
        }
      }
      // row max over the row's kSplit parts
      const int slot = (t % 3) * kBM + row;
      atomicMax(mslot + slot, ordered(__float_as_int(mx)));
      asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "n"(kBarThreads) : "memory");
      mx = __int_as_float(ordered(mslot[slot])) * sl2;
      if (part == 0) mslot[((t + 2) % 3) * kBM + row] = kNegInf;
      if (!alive) continue;
      if (kBias && bias_smem) {  // the tile's bias row lands with V_t
        alive = mbar_wait_warp(v_full + t % C::kVStages, (t / C::kVStages) & 1, abort_flag);
        if (!alive) continue;
      }
      bool rescale = false;
      float alpha = 1.f;
      if (first) {
        m = mx;
      } else if (mx > m + kRescaleThreshold) {
        alpha = fast_exp2(m - mx);
        m = mx;
        rescale = true;
      }
      const uint64_t sl2x2 = pack_f2(sl2, sl2), negm2 = pack_f2(-m, -m);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
      uint32_t pk[kCols / 2];
      if (kBias && brow) {
        // y = s * scale * log2e + (bias * log2e - m); columns past the segment's end are -inf in r
        constexpr float kLog2e = 1.4426950408889634f;
        const uint64_t l2e2 = pack_f2(kLog2e, kLog2e);
        const bool full = lim >= kCols;
        const uint32_t bs = bias_smem ? smem_u32(brow) : 0u;
#pragma unroll
        for (int j = 0; j < kCols; j += 4) {
          float4 bq;
          if (bias_smem) {
            bq = lds_f4(bs + j * 4);
          } else if (full) {
            bq = __ldg(reinterpret_cast<const float4*>(brow + j));
          } else {
            bq.x = j < lim ? __ldg(brow + j) : 0.f;
            bq.y = j + 1 < lim ? __ldg(brow + j + 1) : 0.f;
            bq.z = j + 2 < lim ? __ldg(brow + j + 2) : 0.f;
            bq.w = j + 3 < lim ? __ldg(brow + j + 3) : 0.f;
          }
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int jj = j + 2 * h2;
            const uint64_t c2 = fma_f2(h2 ? pack_f2(bq.z, bq.w) : pack_f2(bq.x, bq.y), l2e2, negm2);
            const uint64_t y = fma_f2(pack_f2(__uint_as_float(r[jj]), __uint_as_float(r[jj + 1])), sl2x2, c2);
            float y0, y1;
            unpack_f2(y, y0, y1);
            const float p0 = fast_exp2(y0), p1 = fast_exp2(y1);
            acc[(jj >> 1) & 3] = add_f2(acc[(jj >> 1) & 3], pack_f2(p0, p1));
            pk[jj >> 1] = pack_bf16x2(p0, p1);
          }
        }
      } else {
        // exponent arguments two at a time (f32x2 FMA), exp2 on the XU pipe, row sum in four packed
        // accumulators (f32x2 adds), P packed to bf16 pairs
#pragma unroll
        for (int j = 0; j < kCols; j += 2) {
          const uint64_t y = fma_f2(pack_f2(__uint_as_float(r[j]), __uint_as_float(r[j + 1])), sl2x2, negm2);
          float y0, y1;
          unpack_f2(y, y0, y1);
          const float p0 = fast_exp2(y0), p1 = fast_exp2(y1);
          acc[(j >> 1) & 3] = add_f2(acc[(j >> 1) & 3], pack_f2(p0, p1));
          pk[j >> 1] = pack_bf16x2(p0, p1);
        }
      }
      float a0, a1, a2, a3, a4, a5, a6, a7;
      unpack_f2(acc[0], a0, a1);
      unpack_f2(acc[1], a2, a3);
      unpack_f2(acc[2], a4, a5);
      unpack_f2(acc[3], a6, a7);
      l = l * alpha + (((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7)));
      tmem_st_n<kCols / 2>(s_addr + part * (kCols / 2), pk);
      // tcgen05.ld/st are warp-collective: the warp rescales together if any of its rows needs it
      // (alpha == 1 on the rows that do not).  Only then must PV_{t-1} be complete; P_t goes to the
      // MMA without waiting for it (the tensor core runs PV_{t-1} before PV_t).  S_t complete
      // implies PV_{t-2}, hence PV_{t-3}, complete, and PV_{t+1} needs this warp's p_ready, so the
      // parity wait on o_done[(t-1) % 2] for PV_{t-1} cannot alias.
      if (__any_sync(0xffffffffu, rescale)) {
        if (t > 0) alive = mbar_wait_warp(o_done + ((t - 1) & 1), ((t - 1) >> 1) & 1, abort_flag);
      }
      if (!alive) continue;
      if (__any_sync(0xffffffffu, rescale)) {
        tc_fence_after();
        const uint32_t o_addr = tmem + lane_addr + 256 + (t >= T1 ? HD : 0) + part * kOCols;
#pragma unroll
        for (int c = 0; c < kOCols / kOC; ++c) {
          uint32_t o[kOC];
          tmem_ld_n<kOC>(o_addr + c * kOC, o);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < kOC; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
          tmem_st_n<kOC>(o_addr + c * kOC, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_ready + b);  // one arrival per warp, after the whole warp's stores
    }
    if (alive && T > 0) alive = mbar_wait_warp(o_final, 0, abort_flag);
    const bool ok = alive;
    // partial row sums of the row's parts, exchanged through the K ring: o_final has seen every MMA
    // complete, and every load the MMAs waited for, so no copy or MMA touches the ring any more
    float* xchg = reinterpret_cast<float*>(smem + C::kOffK);
    const bool has_hist = p.tiles[2] > 0;
    if (!has_hist) {
      m_loc = m;
      l_loc = l;
    }
    xchg[part * kBM + row] = l_loc;
    xchg[(kSplit + part) * kBM + row] = l;
    asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "n"(kBarThreads) : "memory");
    float l_loc_row = xchg[row], l_hist_row = xchg[kSplit * kBM + row];
#pragma unroll
    for (int i = 1; i < kSplit; ++i) {  // fixed order: the same sum on every run
      l_loc_row += xchg[i * kBM + row];
      l_hist_row += xchg[(kSplit + i) * kBM + row];
    }
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
      const uint32_t oa_addr = tmem + lane_addr + 256 + part * kOCols;
      const uint32_t ob_addr = oa_addr + HD;
      // Output tiles staged in the free K/V rings, as the 128-byte-swizzled {64 cols, 128 rows} boxes
      // of the bulk tensor stores: O_loc and O_full in the V ring, D in the second K stage (the
      // first holds the row-sum exchange).
      auto put = [&](int which, int col, const float* v8) {  // 8 values at tile column col
        uint4 w;
        w.x = pack_bf16x2(v8[0], v8[1]);
        w.y = pack_bf16x2(v8[2], v8[3]);
        w.z = pack_bf16x2(v8[4], v8[5]);
        w.w = pack_bf16x2(v8[6], v8[7]);
        const int box = col >> 6, q = (col & 63) >> 3;
        *reinterpret_cast<uint4*>(stage_out_base<HD>(smem, which) + box * (kBM * 128) + row * 128 +
                                  ((q ^ (row & 7)) << 4)) = w;
      };
#pragma unroll 1
      for (int c = 0; c < kOCols / kEC; ++c) {
        uint32_t oa[kEC], ob[kEC];
        tmem_ld_n<kEC>(oa_addr + c * kEC, oa);
        if (has_hist) tmem_ld_n<kEC>(ob_addr + c * kEC, ob);
        tmem_wait_ld();
        float vl[kEC], vf[kEC], vd[kEC];
#pragma unroll
        for (int j = 0; j < kEC; ++j) {
          vl[j] = __uint_as_float(oa[j]) * inv_l_loc;
          vf[j] = has_hist ? fmaf(w_loc, vl[j], w_hist * (__uint_as_float(ob[j]) * inv_l_hist)) : vl[j];
          vd[j] = vf[j] - vl[j];
        }
#pragma unroll
        for (int i = 0; i < kEC / 8; ++i) {
          const int col = part * kOCols + c * kEC + 8 * i;
          put(0, col, vl + 8 * i);
          put(1, col, vf + 8 * i);
          if (p.d_out) put(2, col, vd + 8 * i);
        }
      }
      if (live && part == 0) {
        const float ln2 = 0.69314718055994531f;
        p.lse_loc[(long long)head * p.n_q + grow] = lse_loc2 * ln2;
        p.lse_hist[(long long)head * p.n_q + grow] = has_hist ? lse_hist2 * ln2 : -INFINITY;
      }
      fence_proxy_async_smem_attn();
    }
    // every softmax thread has staged its part (or the CTA gave up); one thread stores the tiles and
    // waits until the bulk copies have read shared memory
    asm volatile("bar.sync 5, %0;" ::"n"(kSoftmaxThreads) : "memory");
    if (warp == kFirstSoftmaxWarp && lane == 0 && !*abort_flag) {
      const int n_out = p.d_out ? 3 : 2;
      for (int w = 0; w < n_out; ++w)
        for (int b = 0; b < HD / 64; ++b)
          store_tile_2d(&maps.out[w], stage_out_base<HD>(smem, w) + b * (kBM * 128), head * HD + 64 * b, q0);
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
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
  for (int s = 0; s < 3; ++s)  // vector loads of each part's biases
    if (a.bias[s] && a.n_kv[s] > 0 && (!al16(a.bias[s]) || (a.ld_bias[s] % 4))) return false;
  return true;
}

template <int HD, bool kBias>
static cudaError_t launch_hd(const AttnLaunch& a, cudaStream_t stream, int* n_launched) {
  constexpr int kSplit = kBias ? 4 : 2;
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
  if (!make_map_bf16_2d(&maps.out[0], a.o_loc, a.n_q, d, a.ld_o, 64, kBM) ||
      !make_map_bf16_2d(&maps.out[1], a.o_full, a.n_q, d, a.ld_o, 64, kBM) ||
      (a.d_out && !make_map_bf16_2d(&maps.out[2], a.d_out, a.n_q, d, a.ld_o, 64, kBM)))
    return cudaErrorInvalidValue;
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
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<HD, kBias, kSplit>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>((a.n_q + kBM - 1) / kBM), static_cast<unsigned>(a.n_heads));
  attn_tc_kernel<HD, kBias, kSplit><<<grid, threads_for(kSplit), C::kSmemBytes, stream>>>(maps, p);
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
