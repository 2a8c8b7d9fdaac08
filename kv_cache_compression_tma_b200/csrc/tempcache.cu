// tempcache.cu -- FAST-AR TempCache on sm_100a: top-1 matching of a new frame's keys against a
// merged KV cache (tcgen05 tensor cores) and the merge itself (CUDA cores).
//
// FAST-AR page, section 2 "Core components", A (TempCache) with Lemma 5.1: tokens of a new frame
// that correspond to a cached token are merged into it; merging identical keys is exact when the
// group's values are averaged and its logit is shifted by the log of the group size.  This library
// keeps, per head, entries with a representative key, the mean value of the group, the group size
// (count), ln(count) as the attention logit bias (-inf for an empty slot) and the inverse norm of
// the key (-1 for an empty slot).  A new token joins its best entry when the cosine similarity of the
// keys reaches a threshold; the others are appended after the head's last entry in token order.
//
// Match kernel: one CTA per (128 new tokens, head).  Warp 0 loads the new-key tile once and the
// cache-key tiles (128 entries) through a 4-slot TMA ring; warp 1 issues S = K_new K_cache^T
// (tcgen05.mma kind::f16, bf16 -> fp32 in TMEM, two S buffers); warps 2..5 (thread = new token =
// TMEM lane) keep a running maximum of S_j * invnorm_j over the live entries (first maximum wins),
// and write the entry and its cosine similarity (times the token's own inverse norm).
// Merge kernel: one CTA per head; merged (entry, token) pairs are sorted in shared memory (bitonic),
// so every group's members are summed in token order (deterministic); unmatched tokens get their
// slots from a prefix count.
#include <math.h>
#include <string.h>

#include "internal.h"
#include "sm100.cuh"

namespace ispa {
namespace {

constexpr int kBM = 128, kBN = 128;
constexpr int kThreads = 192;
constexpr int kSlots = 4;

template <int HD>
struct MCfg {
  static constexpr int kBoxes = HD / 64;
  static constexpr int kBoxBytes = 128 * 128;
  static constexpr int kTileBytes = kBM * HD * 2;
  static constexpr int kOffK = kTileBytes;
  static constexpr int kOffBar = kOffK + kSlots * kTileBytes;
  static constexpr int kNumBars = 1 + 2 * kSlots + 2 + 2 + 1;  // q, full, empty, s_full[2], s_free[2], final
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, kBN, false, false);
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct MatchParams {
  int n_new, n_cache;
  const float* inv_norm;  // [H, n_cache] (row stride ld_state)
  long long ld_state;
  int* idx;               // [H, n_new]
  float* sim;
  unsigned* status;
};

template <int HD>
__global__ void __launch_bounds__(kThreads, 1)
    tc_match_kernel(const __grid_constant__ CUtensorMap map_new, const __grid_constant__ CUtensorMap map_cache,
                    const MatchParams p) {
  using C = MCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* full = q_full + 1;
  uint64_t* empty = full + kSlots;
  uint64_t* s_full = empty + kSlots;   // [2] S buffer holds a tile
  uint64_t* s_free = s_full + 2;       // [2] the four row warps have read it
  uint64_t* final_bar = s_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  volatile int* never = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 8);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.y;
  const int t0 = blockIdx.x * kBM;
  const int T = (p.n_cache + kBN - 1) / kBN;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(s_free + i, 4);
    }
    mbar_init(final_bar, 1);
    *abort_flag = 0;
    *never = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, C::kTileBytes);
#pragma unroll
      for (int b = 0; b < C::kBoxes; ++b)
        tma_load_2d(smem + b * C::kBoxBytes, &map_new, q_full, head * HD + 64 * b, t0);
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const int s = t % kSlots;
        if (t >= kSlots && !mbar_wait(empty + s, ((t / kSlots) - 1) & 1, abort_flag)) {
          atomicOr(p.status, kStatusTimeout);
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(full + s, C::kTileBytes);
#pragma unroll
        for (int b = 0; b < C::kBoxes; ++b)
          tma_load_2d(smem + C::kOffK + s * C::kTileBytes + b * C::kBoxBytes, &map_cache, full + s, head * HD + 64 * b,
                      t * kBN);
        issued = t + 1;
      }
      if (*abort_flag) {
        for (int t = issued - 1; t >= 0 && t >= issued - kSlots; --t)
          mbar_wait(full + t % kSlots, (t / kSlots) & 1, never);
        mbar_wait(q_full, 0, never);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0, abort_flag);
      tc_fence_after();
      const uint32_t qb = smem_u32(smem);
      for (int t = 0; ok && t < T; ++t) {
        const int s = t % kSlots, b = t & 1;
        if (!mbar_wait(full + s, (t / kSlots) & 1, abort_flag) ||
            (t >= 2 && !mbar_wait(s_free + b, ((t >> 1) - 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t kb = smem_u32(smem + C::kOffK + s * C::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kBoxBytes + (kk & 3) * 32;
          umma_ss(tmem + b * 128, sw128_desc(qb + off, 16, 1024), sw128_desc(kb + off, 16, 1024), C::kIdesc,
                  kk > 0 ? 1u : 0u);
        }
        umma_commit(s_full + b);
        umma_commit(empty + s);
      }
      if (!ok) {
        atomicOr(p.status, kStatusTimeout);
        *abort_flag = 1;
      }
      umma_commit(final_bar);
      mbar_wait(final_bar, 0, never);
    }
  } else {
    // thread = new token (TMEM lane); its own inverse norm from the staged tile (128-byte swizzle:
    // row r's 16-byte chunk c sits at chunk c ^ (r & 7))
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    bool alive = mbar_wait_warp(q_full, 0, abort_flag);
    float rn = 0.f;
    if (alive) {
      float ss = 0.f;
#pragma unroll
      for (int b = 0; b < C::kBoxes; ++b) {
        const uint8_t* rowp = smem + b * C::kBoxBytes + row * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 w = *reinterpret_cast<const uint4*>(rowp + ((c ^ (row & 7)) << 4));
          const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float lo = __uint_as_float(u[i] << 16), hi = __uint_as_float(u[i] & 0xFFFF0000u);
            ss = fmaf(lo, lo, fmaf(hi, hi, ss));
          }
        }
      }
      rn = ss > 0.f ? rsqrtf(ss) : 0.f;
    }
    float best = -INFINITY;
    int best_j = -1;
    const float* wrow = p.inv_norm + static_cast<long long>(head) * p.ld_state;
    for (int t = 0; alive && t < T; ++t) {
      const int b = t & 1;
      alive = mbar_wait_warp(s_full + b, (t >> 1) & 1, abort_flag);
      if (!alive) break;
      tc_fence_after();
      const int key0 = t * kBN;
      const int valid = min(kBN, p.n_cache - key0);
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t sv[32];
        tmem_ld32(tmem + lane_addr + b * 128 + c * 32, sv);
        float w[32];
        if (valid == kBN) {
          const float4* w4 = reinterpret_cast<const float4*>(wrow + key0 + c * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 x = __ldg(w4 + i);
            w[4 * i] = x.x;
            w[4 * i + 1] = x.y;
            w[4 * i + 2] = x.z;
            w[4 * i + 3] = x.w;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) w[i] = c * 32 + i < valid ? __ldg(wrow + key0 + c * 32 + i) : -1.f;
        }
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float cs = w[i] >= 0.f ? __uint_as_float(sv[i]) * w[i] : -INFINITY;
          if (cs > best) {
            best = cs;
            best_j = key0 + c * 32 + i;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free + b);
    }
    if (!alive) {
      atomicOr(p.status, kStatusTimeout);
      *abort_flag = 1;
    } else if (t0 + row < p.n_new) {
      const long long o = static_cast<long long>(head) * p.n_new + t0 + row;
      p.idx[o] = best_j;
      p.sim[o] = best_j >= 0 ? best * rn : -INFINITY;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ------------------------------------------------------------------------------------------ merge
constexpr int kMergeThreads = 512;
constexpr int kMaxNew = 4096;  // tokens of one frame handled by one CTA's shared-memory sort

struct MergeParams {
  int n_heads, hd, n_new, n_cache;
  long long ld_cache, ld_new, ld_state;
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
  int* count;
  float* bias;
  float* inv_norm;
  int* n_valid;
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  const int* idx;
  const float* sim;
  float threshold;
  unsigned* status;
};

__global__ void __launch_bounds__(kMergeThreads) tc_merge_kernel(const MergeParams p) {
  __shared__ uint32_t key[kMaxNew];
  __shared__ int rank[kMaxNew];
  __shared__ int warp_tot[kMergeThreads / 32];
  __shared__ int s_n0;
  const int h = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kWarps = kMergeThreads / 32;
  const int T = p.n_new;
  int n_pow2 = 1;
  while (n_pow2 < T) n_pow2 <<= 1;
  if (tid == 0) {
    int n0 = p.n_valid[h];
    if (n0 < 0 || n0 > p.n_cache) {  // the caller's bound on the live entries was wrong
      atomicOr(p.status, kStatusInternal);
      n0 = n0 < 0 ? 0 : p.n_cache;
    }
    s_n0 = n0;
  }
  __syncthreads();
  const int n0 = s_n0;
  const int* idx = p.idx + static_cast<long long>(h) * T;
  const float* sim = p.sim + static_cast<long long>(h) * T;
  // merged tokens as sortable (entry, token) keys; the rest sort to the end
  for (int t = tid; t < n_pow2; t += kMergeThreads) {
    uint32_t k = 0xFFFFFFFFu;
    if (t < T) {
      const int e = idx[t];
      if (e >= 0 && e < n0 && sim[t] >= p.threshold) k = (static_cast<uint32_t>(e) << 12) | static_cast<uint32_t>(t);
    }
    key[t] = k;
  }
  __syncthreads();
  for (int size = 2; size <= n_pow2; size <<= 1) {  // bitonic sort, ascending
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < n_pow2; i += kMergeThreads) {
        const int j = i ^ stride;
        if (j > i) {
          const bool up = (i & size) == 0;
          const uint32_t a = key[i], b = key[j];
          if ((a > b) == up) {
            key[i] = b;
            key[j] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  // groups: a warp per run of equal entries, members summed in token order
  const long long lds = p.ld_state;
  const int hd = p.hd;
  for (int i = warp; i < T; i += kWarps) {
    const uint32_t k = key[i];
    if (k == 0xFFFFFFFFu) continue;
    const uint32_t e = k >> 12;
    if (i > 0 && (key[i - 1] >> 12) == e && key[i - 1] != 0xFFFFFFFFu) continue;  // not the run's start
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    int n = 0;
    for (int j = i; j < T && key[j] != 0xFFFFFFFFu && (key[j] >> 12) == e; ++j, ++n) {
      const int t = static_cast<int>(key[j] & 0xFFFu);
      const __nv_bfloat16* vr = p.v_new + static_cast<long long>(t) * p.ld_new + static_cast<long long>(h) * hd;
      for (int c = lane, q = 0; c < hd; c += 32, ++q) acc[q] += __bfloat162float(vr[c]);
    }
    const int g = p.count[h * lds + e];
    __nv_bfloat16* ve = p.v_cache + static_cast<long long>(e) * p.ld_cache + static_cast<long long>(h) * hd;
    for (int c = lane, q = 0; c < hd; c += 32, ++q)
      ve[c] = __float2bfloat16_rn((static_cast<float>(g) * __bfloat162float(ve[c]) + acc[q]) / static_cast<float>(g + n));
    if (lane == 0) {
      p.count[h * lds + e] = g + n;
      p.bias[h * lds + e] = logf(static_cast<float>(g + n));
    }
  }
  // unmatched tokens: slots n0 + (their rank in token order)
  for (int t = tid; t < kMaxNew; t += kMergeThreads) rank[t] = 0;
  __syncthreads();
  const int per = (T + kMergeThreads - 1) / kMergeThreads;  // contiguous tokens per thread
  int local = 0;
  for (int q = 0; q < per; ++q) {
    const int t = tid * per + q;
    if (t < T) {
      const int e = idx[t];
      const bool merged = e >= 0 && e < n0 && sim[t] >= p.threshold;
      rank[t] = merged ? -1 : local;
      local += merged ? 0 : 1;
    }
  }
  // exclusive scan of the per-thread counts
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int base = 0;
  for (int w = 0; w < warp; ++w) base += warp_tot[w];
  const int excl = base + incl - local;
  for (int q = 0; q < per; ++q) {
    const int t = tid * per + q;
    if (t < T && rank[t] >= 0) rank[t] += excl;
  }
  int total = 0;
  for (int w = 0; w < kWarps; ++w) total += warp_tot[w];
  __syncthreads();
  // copy the unmatched tokens (a warp per token)
  for (int t = warp; t < T; t += kWarps) {
    const int r = rank[t];
    if (r < 0) continue;
    const int slot = n0 + r;
    const long long src = static_cast<long long>(t) * p.ld_new + static_cast<long long>(h) * hd;
    const long long dst = static_cast<long long>(slot) * p.ld_cache + static_cast<long long>(h) * hd;
    float ss = 0.f;
    for (int c = lane; c < hd; c += 32) {
      const __nv_bfloat16 kv = p.k_new[src + c];
      p.k_cache[dst + c] = kv;
      p.v_cache[dst + c] = p.v_new[src + c];
      const float f = __bfloat162float(kv);
      ss = fmaf(f, f, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) {
      p.count[h * lds + slot] = 1;
      p.bias[h * lds + slot] = 0.f;
      p.inv_norm[h * lds + slot] = ss > 0.f ? rsqrtf(ss) : 0.f;
    }
  }
  // empty slots up to the caller's next bound: no weight, zero keys and values
  const int n1 = n0 + total, bound = p.n_cache + T;
  for (int e = n1 + warp; e < bound; e += kWarps) {
    const long long dst = static_cast<long long>(e) * p.ld_cache + static_cast<long long>(h) * hd;
    for (int c = lane; c < hd; c += 32) {
      p.k_cache[dst + c] = __float2bfloat16_rn(0.f);
      p.v_cache[dst + c] = __float2bfloat16_rn(0.f);
    }
    if (lane == 0) {
      p.count[h * lds + e] = 0;
      p.bias[h * lds + e] = -INFINITY;
      p.inv_norm[h * lds + e] = -1.f;
    }
  }
  if (tid == 0) p.n_valid[h] = n1;
}

}  // namespace

cudaError_t launch_tc_match(const TcMatchLaunch& a, cudaStream_t s, int* n_launched) {
  if (a.n_new == 0) return cudaSuccess;
  CUtensorMap mn, mc;
  memset(&mn, 0, sizeof(mn));
  memset(&mc, 0, sizeof(mc));
  const uint64_t d = static_cast<uint64_t>(a.n_heads) * a.head_dim;
  if (!make_map_bf16_2d(&mn, a.k_new, a.n_new, d, a.ld_new, 64, kBM)) return cudaErrorInvalidValue;
  if (a.n_cache == 0)  // no cache tile is loaded: every token gets idx -1, sim -inf
    mc = mn;
  else if (!make_map_bf16_2d(&mc, a.k_cache, a.n_cache, d, a.ld_cache, 64, kBN))
    return cudaErrorInvalidValue;
  MatchParams p;
  p.n_new = static_cast<int>(a.n_new);
  p.n_cache = static_cast<int>(a.n_cache);
  p.inv_norm = a.inv_norm;
  p.ld_state = a.ld_state;
  p.idx = a.idx;
  p.sim = a.sim;
  p.status = a.status;
  dim3 grid(static_cast<unsigned>((a.n_new + kBM - 1) / kBM), static_cast<unsigned>(a.n_heads));
  cudaError_t e;
  if (a.head_dim == 128) {
    e = cudaFuncSetAttribute(tc_match_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, MCfg<128>::kSmemBytes);
    if (e == cudaSuccess) tc_match_kernel<128><<<grid, kThreads, MCfg<128>::kSmemBytes, s>>>(mn, mc, p);
  } else {
    e = cudaFuncSetAttribute(tc_match_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, MCfg<64>::kSmemBytes);
    if (e == cudaSuccess) tc_match_kernel<64><<<grid, kThreads, MCfg<64>::kSmemBytes, s>>>(mn, mc, p);
  }
  if (e != cudaSuccess) return e;
  *n_launched += 1;
  return cudaGetLastError();
}

bool tc_merge_supported(int64_t n_new) { return n_new <= kMaxNew; }

cudaError_t launch_tc_merge(const TcMergeLaunch& a, cudaStream_t s, int* n_launched) {
  if (a.n_new == 0) return cudaSuccess;
  MergeParams p;
  p.n_heads = a.n_heads;
  p.hd = a.head_dim;
  p.n_new = static_cast<int>(a.n_new);
  p.n_cache = static_cast<int>(a.n_cache);
  p.ld_cache = a.ld_cache;
  p.ld_new = a.ld_new;
  p.ld_state = a.ld_state;
  p.k_cache = static_cast<__nv_bfloat16*>(a.k_cache);
  p.v_cache = static_cast<__nv_bfloat16*>(a.v_cache);
  p.count = a.count;
  p.bias = a.bias;
  p.inv_norm = a.inv_norm;
  p.n_valid = a.n_valid;
  p.k_new = static_cast<const __nv_bfloat16*>(a.k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(a.v_new);
  p.idx = a.idx;
  p.sim = a.sim;
  p.threshold = a.threshold;
  p.status = a.status;
  tc_merge_kernel<<<a.n_heads, kMergeThreads, 0, s>>>(p);
  *n_launched += 1;
  return cudaGetLastError();
}

}  // namespace ispa
