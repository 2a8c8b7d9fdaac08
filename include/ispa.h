/*
 * ispa.h -- C ABI of the ISPA hot path on NVIDIA B200 (sm_100a).
 *
 * ISPA ("Instance-Specific Parametric Absorption (ISPA) for Memory-Efficient Video Generation",
 * technical summary, section 2 "Methodology") runs a streaming video generator in three stages:
 *   1. dual-stream warmup: every layer computes, in one attention pass, the output over the local
 *      context only (A_loc: sink tokens + current chunk) and the output over the full history
 *      (A_full), by tracking log-sum-exp per branch and merging the branches post-hoc;
 *   2. layer absorb at T_warm: dW = (A_loc^T A_loc + lam I)^-1 A_loc^T (A_full - A_loc) W, the
 *      closed-form minimiser of ||A_loc (W + dW) - A_full W||^2 + lam ||dW||^2;
 *   3. the K layers with the lowest reconstruction error eps become local-only layers that use
 *      W_new = W + dW ("Dynamic Layer Selection").
 *
 * Conventions for every call:
 *   - Every pointer argument of a device call is DEVICE memory allocated and owned by the caller,
 *     unless the comment says "host".  The library never frees caller memory and makes no device
 *     allocation on any call.  What it owns: (a) module-scope device variables, which the CUDA
 *     runtime places on every device that loads the library and keeps until the process exits --
 *     one uint32 status word per device, and the scratch array of ispa_absorb_static (36.8 MiB);
 *     (b) six CUDA streams and a few hundred events per device, created by the first ispa_absorb
 *     call on that device and kept until exit.
 *   - Device addresses of those variables are resolved once per device and cached for the life of
 *     the process: they assume the device's primary context is never reset or destroyed while the
 *     library is loaded (no cudaDeviceReset between calls).
 *   - `stream` is a cudaStream_t passed as an opaque pointer (NULL = the legacy default stream).
 *     Device calls are asynchronous on that stream; the outputs are valid once it is synchronised.
 *   - Argument, shape, dtype and alignment errors are detected on the host before anything is
 *     launched and return ISPA_ERR_INVALID_ARG or ISPA_ERR_UNSUPPORTED; a launch failure returns
 *     ISPA_ERR_CUDA.  Conditions found on the device (non-SPD system, non-finite values, a bounded
 *     wait that ran out) set bits of the sticky per-device status word, read and cleared by
 *     ispa_get_device_status().  No kernel traps.
 *   - Matrices are row-major.  "ld" arguments are row strides in elements.
 */
#ifndef ISPA_H
#define ISPA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ISPA_API __attribute__((visibility("default")))
#else
#define ISPA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ISPA_OK = 0,
  ISPA_ERR_INVALID_ARG = 1,  /* bad pointer, size, stride, flag or alignment                      */
  ISPA_ERR_UNSUPPORTED = 2,  /* valid request this build has no kernel for                        */
  ISPA_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed                              */
  ISPA_ERR_NOT_SPD = 4,      /* device: a Cholesky pivot of G + lam I was <= 0 or not finite      */
  ISPA_ERR_NONFINITE = 5,    /* device: NaN/Inf met in an output of the absorb (dW or eps)        */
  ISPA_ERR_TIMEOUT = 6,      /* device: a bounded barrier wait ran out; outputs are undefined     */
  ISPA_ERR_INTERNAL = 7      /* device: a kernel found its launch unusable (e.g. a shared-memory  */
                             /* base without the alignment its layouts need); nothing computed     */
} ispa_status;

typedef enum { ISPA_BF16 = 0, ISPA_F32 = 1 } ispa_dtype;

/* Segment indices of ispa_attn_args.n_kv / k / v. */
enum { ISPA_SEG_SINK = 0, ISPA_SEG_LOCAL = 1, ISPA_SEG_HIST = 2 };

/*
 * Decomposable (dual-stream) attention, ISPA section 2, stage 1 ("Decomposable Attention" over
 * online-softmax / log-sum-exp state; contribution 2).
 *
 * For every head h and query row i, with s_j = softmax_scale * q_i . k_j:
 *   local branch   keys j in sink + local:  O_loc = softmax(s) V,  lse_loc  = log sum_j exp(s_j)
 *   history branch keys j in hist:           O_hist (internal),      lse_hist = log sum_j exp(s_j)
 *   post-hoc merge O_full = sigma(lse_loc - lse_hist) O_loc + sigma(lse_hist - lse_loc) O_hist,
 * i.e. O_full is exact softmax attention over sink + local + hist.  Both branches come out of ONE
 * pass over the keys.  No mask (bidirectional within the chunk; the cache holds only past chunks).
 * lse values are natural logs of the scaled logits.  n_kv[ISPA_SEG_HIST] == 0 gives
 * lse_hist = -inf and O_full bitwise equal to O_loc (and D == 0).
 *
 * Layout: q and every k/v segment are [tokens, n_heads, head_dim] with token stride ld_* elements
 * (>= n_heads*head_dim); outputs o_loc, o_full, d_out are [n_q, n_heads*head_dim] with row stride
 * ld_o, i.e. the A matrices of stage 2 (one row per query token, heads concatenated).
 * lse_loc / lse_hist are fp32 [n_heads, n_q].  d_out (optional, NULL to skip) receives
 * D = O_full - O_loc formed in fp32 before rounding to dtype; it is the input of ispa_accum_stats.
 *
 * Kernels: dtype ISPA_BF16 runs the tcgen05/TMEM tensor-core kernel (bf16 MMA, fp32 accumulation,
 * P rounded to bf16 for the PV product); it needs head_dim 64 or 128, 16-byte aligned base pointers
 * and strides that are multiples of 8.  A bf16 call outside those rules returns
 * ISPA_ERR_UNSUPPORTED and launches nothing, unless flags has ISPA_ATTN_CUDA_CORES, which asks for
 * the CUDA-core kernel (fp32 arithmetic, head_dim 16, 32, 64 or 128, any alignment) explicitly.
 * ISPA_F32 always runs the CUDA-core kernel (the only fp32 kernel).
 * Requires n_q >= 0, n_kv[SINK] + n_kv[LOCAL] >= 1, n_heads >= 1.
 *
 * kv_bias (FAST-AR page, section 2 A "TempCache", Lemma 5.1): a segment may carry an additive logit
 * bias per key, in natural-log units: the score of key j of head h becomes
 * softmax_scale * q.k_j + kv_bias[s][h * ld_bias[s] + j].  A merged cache passes the log of each
 * entry's group size (-inf for an empty slot, which then takes no weight).  The kernel takes the
 * running maximum over the unbiased scores and applies the bias inside the exponent, so finite
 * biases must lie in [-64, 16] (a group of up to e^16 members); -inf excludes a key.  Tensor-core
 * kernel only (16-byte aligned bias, ld_bias a multiple of 4); with ISPA_ATTN_CUDA_CORES or ISPA_F32
 * a bias returns ISPA_ERR_UNSUPPORTED.  Every query row needs at least one key of finite bias in
 * sink + local.
 */
#define ISPA_ATTN_CUDA_CORES 0x1

typedef struct {
  int32_t dtype;          /* ispa_dtype of q, k, v, o_loc, o_full, d_out                        */
  int32_t n_heads;
  int32_t head_dim;
  int32_t flags;          /* 0, or ISPA_ATTN_CUDA_CORES to run the CUDA-core kernel on any case */
  int64_t n_q;            /* query tokens of the current chunk                                 */
  int64_t n_kv[3];        /* key/value tokens per segment: sink, local (current chunk), history  */
  const void* q;
  int64_t ld_q;
  const void* k[3];
  const void* v[3];
  int64_t ld_k[3];
  int64_t ld_v[3];
  float softmax_scale;    /* 0 selects 1/sqrt(head_dim)                                          */
  float reserved0;
  void* o_loc;            /* out [n_q, d]                                                        */
  void* o_full;           /* out [n_q, d]                                                        */
  int64_t ld_o;
  float* lse_loc;         /* out [n_heads, n_q]                                                  */
  float* lse_hist;        /* out [n_heads, n_q]                                                  */
  void* d_out;            /* optional out [n_q, d] (row stride ld_o); NULL skips it              */
  const float* kv_bias[3];/* optional per-key logit bias of each segment, fp32 [n_heads, n_kv[s]]  */
  int64_t ld_bias[3];     /* (row stride ld_bias[s] >= n_kv[s]); NULL = no bias                    */
} ispa_attn_args;

ISPA_API ispa_status ispa_dual_stream_attn(const ispa_attn_args* args, void* stream);

/*
 * Warmup sufficient statistics, ISPA section 2, stage 2: the two factors of the closed form,
 *   G += A_loc^T A_loc,   R += A_loc^T D,   and   S += D^T D   (D = A_full - A_loc),
 * accumulated over the rows of one call (m rows of width d).  S is not on the pages: it lets the
 * reconstruction error be evaluated from statistics alone in ispa_absorb.
 *
 * a_loc, a_second: dtype [m, d] with row stride lda.  a_second is D by default (as written by
 * ispa_dual_stream_attn's d_out); with ISPA_STATS_SECOND_IS_FULL it is A_full and the kernel forms
 * the D products itself (exactly, from the two bf16 operands).  G, R, S: fp32 [d, d], row stride d,
 * all entries written (G and S in full, both triangles).  ISPA_STATS_ZERO overwrites instead of
 * accumulating.  m == 0 is a no-op (or zero-fill with ISPA_STATS_ZERO).
 * bf16 runs the tcgen05 kernel (d a multiple of 128, lda a multiple of 8, 16-byte aligned
 * pointers); other cases run a CUDA-core kernel.
 */
#define ISPA_STATS_ZERO 0x1u
#define ISPA_STATS_SECOND_IS_FULL 0x2u
ISPA_API ispa_status ispa_accum_stats(int32_t dtype, const void* a_loc, const void* a_second, int64_t m,
                             int32_t d, int64_t lda, uint32_t flags, float* G, float* R, float* S,
                             void* stream);

/*
 * Closed-form ridge absorb and reconstruction error, ISPA section 2, stage 2 (objective and closed
 * form) and "Dynamic Layer Selection" (eps).
 *   lam = lambda                     (or lambda * trace(G) / d with ISPA_LAMBDA_REL)
 *   B   = R W ;  G + lam I = L L^T (blocked Cholesky) ;  L Y = B ;  L^T dW = Y
 *         (d < 3072: computed as dW = M^T Y with M = L^-1 from the same forward substitution;
 *          wider layers: blocked back substitution; both substitutions of wide layers go through
 *          the inverses of the 512-wide diagonal blocks of L)
 *   eps = ||A_loc (W + dW) - A_full W||_F^2 evaluated from the statistics:
 *         eps = <W, S W> - 2 <dW, B> + ||Y||_F^2 - lam ||dW||_F^2  (<W, S W> taken as <S, W W^T>),
 *   eps_rel = eps / <W, S W>.
 * G, R, S: fp32 [d, d] (row stride d; only the lower triangles of G and S are read).  W: dtype_w [d, d]
 * as d_in x d_out (y = x W), or d_out x d_in with ISPA_W_TRANSPOSED (the torch Linear layout).
 * dW: out fp32 [d, d] in the d_in x d_out orientation.  eps_out: out device double[4] =
 * {eps, eps_rel, lam, <W, S W>}.  With ISPA_WRITE_WNEW, w_new (dtype_w, same orientation as W,
 * may alias W) receives W + dW rounded to dtype_w.  ws: device workspace of at least
 * ispa_absorb_workspace_size(d) bytes, 256-byte aligned, not used concurrently by another call.
 * A non-positive pivot sets ISPA_ERR_NOT_SPD in the device status word (dW, eps then undefined).
 * d must be a multiple of 16 and at most 16384.
 * Scheduling: the work is enqueued on `stream` and on up to six library-owned streams of the current
 * device (created on first use; the one that carries the factorisation's critical path, and the one
 * that builds the wide layers' block inverses, at the device's highest stream priority), which are
 * joined back into `stream` before the call returns,
 * so every output is ready when `stream` reaches that point.  Enqueues from several host threads on
 * one device are serialised by the library; absorbs that overlap on the GPU need separate workspaces.
 * If the call returns ISPA_ERR_CUDA, part of the work may already be queued on the library streams
 * without having been joined into `stream`: synchronise the device before reusing or freeing the
 * buffers.
 * Workspace: about 7 d^2 floats (ispa_absorb_workspace_size gives the exact figure).
 */
#define ISPA_LAMBDA_REL 0x1u
#define ISPA_W_TRANSPOSED 0x2u
#define ISPA_WRITE_WNEW 0x4u
ISPA_API ispa_status ispa_absorb_workspace_size(int32_t d, size_t* bytes);
ISPA_API ispa_status ispa_absorb(const float* G, const float* R, const float* S, int32_t dtype_w, const void* W,
                        int32_t d, float lambda, uint32_t flags, float* dW, double* eps_out, void* w_new,
                        void* ws, size_t ws_bytes, void* stream);

/*
 * ispa_absorb_static -- the same absorb as ispa_absorb, for callers that cannot allocate device
 * memory.  (Not a step of the ISPA method: the paper has no counterpart; this is a deployment
 * variant of the call above.)
 *
 * Some callers cannot call cudaMalloc or an allocating library routine when the absorb runs: an
 * engine that hands all of its device memory to its own arena up front, a plugin whose host exposes
 * no allocator, or a latency-critical loop that must not pay for an allocation at T_warm.  This entry
 * point therefore takes no workspace: its scratch is a module-scope device array of the library,
 * sized for d <= 1536 (about 36.8 MiB), which every GPU that loads the library holds until the
 * process exits.  The caller still passes G, R, S, W and the outputs dW, eps_out and (optionally)
 * w_new, exactly as for ispa_absorb, and the call allocates nothing.
 *   - d > 1536 returns ISPA_ERR_UNSUPPORTED and launches nothing; use ispa_absorb for wider layers.
 *   - The first call on a device resolves the array's device address (cudaGetSymbolAddress) with
 *     that device current and caches it; make that first call before any stream capture.
 *   - Every call on a device shares the one array and leaves its contents behind; no part of it
 *     needs to start at zero.  Calls whose kernels overlap on the GPU (different streams, or other
 *     threads) race on the array: serialise them.
 */
ISPA_API ispa_status ispa_absorb_static(const float* G, const float* R, const float* S, int32_t dtype_w,
                                        const void* W, int32_t d, float lambda, uint32_t flags, float* dW,
                                        double* eps_out, void* w_new, void* stream);

/*
 * Layer output projection Y = A W, ISPA section 2, stage 3 (memory-efficient inference after
 * T_warm): an L-Layer projects its local-only attention output (ispa_dual_stream_attn with
 * n_kv[ISPA_SEG_HIST] == 0) with W_new = W + dW, an F-Layer its full output with W.
 *   A: dtype [m, d_in], row stride lda.  W: dtype [d_in, d_out] (y = x W), row stride ldw, or with
 *   ISPA_W_TRANSPOSED [d_out, d_in] (the torch Linear layout).  Y: out dtype [m, d_out], row stride
 *   ldy; Y must not overlap A or W.
 * ISPA_BF16 runs a tcgen05 kernel (bf16 products, fp32 accumulation in TMEM, Y rounded once); it
 * needs d_in % 64 == 0, d_out % 128 == 0, 16-byte aligned pointers and strides that are multiples
 * of 8, else ISPA_ERR_UNSUPPORTED.  ISPA_F32 runs an fp32 CUDA-core kernel on any shape.
 * m == 0 is a no-op.
 */
ISPA_API ispa_status ispa_project(int32_t dtype, const void* A, int64_t m, int32_t d_in, int64_t lda, const void* W,
                                  int32_t d_out, int64_t ldw, uint32_t flags, void* Y, int64_t ldy, void* stream);

/*
 * fp8 (E4M3) quantisation for the W8A8 projection, ISPA summary section 4 (results: ISPA combined
 * with W8A8 post-training quantisation).  The pages fix no format; this library's reading is E4M3
 * operands with one fp32 scale per activation row and one per output column of the weight:
 *   s = max |x| / 448 over the row (or column), 1 if that maximum is 0;  q = e4m3(x / s),
 * with an IEEE fp32 division, rounding to the nearest E4M3 value (ties to even) and saturating at
 * +-448 (E4M3: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits, largest finite 448).
 *   X: dtype [rows, cols], row stride ldx elements.  Default: one scale per row, scale[rows] and
 *   q [rows, cols] (row stride ldq bytes).  ISPA_QUANT_COLUMNS: one scale per column, scale[cols],
 *   and q is written TRANSPOSED, [cols, rows] (row stride ldq bytes) -- the K-major layout that
 *   ispa_project_w8a8 takes for the weight, produced from W stored d_in x d_out.  A weight stored in
 *   the torch Linear layout (d_out x d_in) is quantised per row instead, with the same result.
 * Pointers are device memory; rows == 0 or cols == 0 is a no-op.
 */
#define ISPA_QUANT_COLUMNS 0x1u
ISPA_API ispa_status ispa_quantize_e4m3(int32_t dtype, const void* X, int64_t rows, int32_t cols, int64_t ldx,
                                        uint32_t flags, uint8_t* q, int64_t ldq, float* scale, void* stream);

/*
 * W8A8 layer output projection, ISPA summary section 4 with section 2 stage 3 (an L-Layer's output
 * projected by its quantised W_new): Y = diag(sa) (qa qw^T) diag(sw), i.e.
 *   Y_ij = sa_i sw_j sum_k qa_ik qw_jk,
 * with qa E4M3 [m, d_in] (row stride lda bytes) and its row scales sa[m], qw E4M3 [d_out, d_in]
 * (K-major, row stride ldw bytes) and its output-column scales sw[d_out], both as written by
 * ispa_quantize_e4m3.  Products accumulate in fp32 (tcgen05.mma kind::f8f6f4, TMEM); Y is bf16
 * [m, d_out] with row stride ldy elements, rounded once.  Needs d_in % 128 == 0, d_out % 256 == 0,
 * lda and ldw multiples of 16, ldy a multiple of 8 and 16-byte aligned qa, qw, sw and Y, else
 * ISPA_ERR_UNSUPPORTED.  m == 0 is a no-op.
 */
ISPA_API ispa_status ispa_project_w8a8(const uint8_t* qa, const float* sa, int64_t m, int32_t d_in, int64_t lda,
                                       const uint8_t* qw, const float* sw, int32_t d_out, int64_t ldw, void* Y,
                                       int64_t ldy, void* stream);

/*
 * TempCache, FAST-AR page, section 2 "Core components", A, with its Lemma 5.1: the KV cache of a
 * head is compressed by merging each new frame's tokens into the cached tokens they correspond to;
 * merging identical keys is exact when the group's values are averaged and its logit is shifted by
 * the log of the group size.  A merged cache of one segment is, per head h and entry e < capacity:
 *   k_cache, v_cache  bf16 [capacity, n_heads, head_dim] (row stride ld_cache elements): the group's
 *                     representative key (its first member's) and the mean of its members' values;
 *   count     int32 [n_heads, capacity] (row stride ld_state): the group size, 0 for an empty slot;
 *   bias      fp32  [n_heads, capacity] (row stride ld_state): ln(count), -inf for an empty slot --
 *                     pass it as ispa_attn_args.kv_bias of the segment;
 *   inv_norm  fp32  [n_heads, capacity] (row stride ld_state): 1 / ||key|| (0 for a zero key), -1 for
 *                     an empty slot;
 *   n_valid   int32 [n_heads]: the head's entry count (entries 0 .. n_valid-1 are live).
 * A cache starts empty (n_valid = 0) and is built frame by frame with ispa_tempcache_match followed
 * by ispa_tempcache_merge; `n_cache` is the caller's bound on every head's n_valid (the segment length
 * it attends over); after a merge the bound grows by n_new and entries past a head's n_valid up to it
 * are empty (zero key and value, count 0, bias -inf).  Readings of what the page leaves open: the
 * neighbour is the exact top-1 (the page's approximate search in the limit) by cosine similarity of
 * the keys within the same head, ties to the lowest entry; a zero key has similarity 0; the group keeps
 * its first key.
 *
 * ispa_tempcache_match: for every head h and new token t, idx_out[h * n_new + t] = the live entry of
 * largest cosine similarity to k_new[t, h] and sim_out[...] = that similarity (fp32); -1 and -inf when
 * the head has no live entry.  k_new bf16 [n_new, n_heads, head_dim] (row stride ld_new).  Tensor-core
 * kernel: head_dim 64 or 128, 16-byte aligned keys and inv_norm, ld_new / ld_cache multiples of 8,
 * ld_state a multiple of 4.
 */
ISPA_API ispa_status ispa_tempcache_match(int32_t n_heads, int32_t head_dim, const void* k_new, int64_t n_new,
                                          int64_t ld_new, const void* k_cache, int64_t n_cache, int64_t ld_cache,
                                          const float* inv_norm, int64_t ld_state, int32_t* idx_out, float* sim_out,
                                          void* stream);

/*
 * ispa_tempcache_merge: merge a new frame (k_new, v_new bf16 [n_new, n_heads, head_dim], row stride
 * ld_new) into the cache, per head: token t joins entry idx[h, t] when sim[h, t] >= threshold (the
 * entry's value becomes the mean of all its members, rounded to bf16 once per merge, its count and
 * bias grow); the other tokens are appended in token order after the head's last entry.  idx, sim as
 * written by ispa_tempcache_match for the same cache.  Needs capacity >= n_cache + n_new, n_new <=
 * 4096 (else ISPA_ERR_UNSUPPORTED), head_dim a multiple of 32 up to 128.  A head whose n_valid exceeds
 * n_cache sets ISPA_ERR_INTERNAL in the status word (and is clamped).  Deterministic: the members of
 * each group are summed in token order.
 */
ISPA_API ispa_status ispa_tempcache_merge(int32_t n_heads, int32_t head_dim, void* k_cache, void* v_cache,
                                          int64_t ld_cache, int64_t capacity, int64_t n_cache, int32_t* count,
                                          float* bias, float* inv_norm, int64_t ld_state, int32_t* n_valid,
                                          const void* k_new, const void* v_new, int64_t n_new, int64_t ld_new,
                                          const int32_t* idx, const float* sim, float threshold, void* stream);

/*
 * Instance-specific layer selection, ISPA section 2 "Dynamic Layer Selection" (host call, no GPU):
 * rank the n_layers values eps[] (host array) ascending and return the k lowest in idx_out[k]
 * (host), listed in ascending layer index.  Ties go to the lower layer index.  NaN ranks after
 * every number; if a NaN layer is selected the call still fills idx_out and returns
 * ISPA_ERR_NONFINITE.  mask_out (optional host [n_layers]) gets 1 for selected layers, else 0.
 * k == 0 selects nothing; k > n_layers or k < 0 is ISPA_ERR_INVALID_ARG.
 */
ISPA_API ispa_status ispa_select_layers(const double* eps, int32_t n_layers, int32_t k, int32_t* idx_out,
                               uint8_t* mask_out);

/* Synchronises `stream`, then returns and clears the sticky status word of the current device:
 * the most severe of INTERNAL / TIMEOUT / NOT_SPD / NONFINITE seen since the last call (in that
 * order), else ISPA_OK.
 * The word is shared by every stream on the device. */
ISPA_API ispa_status ispa_get_device_status(void* stream);

/*
 * Test hook for the device-status path (not a step of the ISPA method; the pages have no
 * counterpart).  It lets a test make a kernel's bounded waits run out without faulting or hanging
 * the GPU.  flags == 0 (the default) turns every hook off; other bits return ISPA_ERR_INVALID_ARG.
 *   ISPA_TEST_ATTN_NO_LOADS: the tensor-core dual-stream attention kernel issues no TMA loads, so
 *     nothing is ever in flight; each CTA's consumers give up after the bounded wait (about 1 s),
 *     release their tensor memory and return; ispa_get_device_status() then reports
 *     ISPA_ERR_TIMEOUT.  The outputs of such a launch are undefined.
 * The setting is process-wide and read when a kernel is launched.
 */
#define ISPA_TEST_ATTN_NO_LOADS 0x1u
ISPA_API ispa_status ispa_test_set_flags(uint32_t flags);

/* Raw bits of the status word of the current device without clearing it (1 << status). */
ISPA_API ispa_status ispa_peek_device_status_bits(uint32_t* bits_out);

ISPA_API const char* ispa_status_string(ispa_status status);
ISPA_API int32_t ispa_version(void);

/* Number of kernels this library has launched in this process (all devices, all streams). */
ISPA_API uint64_t ispa_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* ISPA_H */
