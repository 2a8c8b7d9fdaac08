"""Plain fp64 CPU oracle for the ISPA hot path.  TEST INFRASTRUCTURE ONLY.

Only the tests, the package's smoke check and the benchmark's CPU-baseline / reference arm may
import this module.  The CUDA library never calls it, and it shares no code with the CUDA path:
both sides only share the seeded input generators in `ispa_inputs`.

What it computes follows the ISPA technical summary ("Instance-Specific Parametric Absorption
(ISPA) for Memory-Efficient Video Generation", section 2 "Methodology", the three-stage "Framework
Core" and "Dynamic Layer Selection"; the same text appears on the Japanese page of the same paper).
The oracle computes the plain definitions, not the fast algorithm:

  * stage 1 (dual-stream warmup): A_loc is attention over the local context only (sink tokens plus
    the current chunk) and A_full is attention over the whole cached history.  The oracle runs them
    as two *separate* naive softmax passes (plus a history-only pass used to check the LSE merge);
  * stage 2 (layer absorb): the ridge objective min ||A_loc (W + dW) - A_full W||^2 + lam ||dW||^2
    and its closed form dW = (A_loc^T A_loc + lam I)^-1 A_loc^T (A_full - A_loc) W, solved by a
    dense LU factorisation with partial pivoting (LAPACK gesv through numpy);
  * layer selection: the reconstruction error eps of every layer, ranked ascending; the K lowest
    become local-attention layers;
  * stage 3: W_new = W + dW, and the layers after T_warm: an L-Layer attends over sink + current
    chunk only (its history K/V are no longer kept) and projects with W_new, an F-Layer attends over
    the full cache and projects with W.

Readings of points the summary leaves open:
  * softmax scale 1/sqrt(head_dim), natural-log LSE of the scaled logits; no mask (attention is
    bidirectional inside a chunk, causal across chunks because the cache holds only past chunks);
  * a row of A is one query token with all heads concatenated (column h*hd + e), so A is [tokens, d]
    and W is the d x d output projection applied as y = A @ W;
  * ||.||_2^2 on matrices is the squared Frobenius norm;
  * lam = lam_rel * trace(G) / d;
  * eps is the data term of the objective at the solved dW (ridge term excluded), reported with
    eps_rel = eps / ||(A_full - A_loc) W||_F^2;
  * ties in the ranking go to the lower layer index, NaN ranks last.

Parity status: every function here is pinned by the CPU tests in tests/test_oracle_pins.py against
closed forms, identities, brute force and textbook routines, except which eps the authors rank by and
its absolute value on synthetic data, which nothing on the pages fixes (parity unpinned for that
reading; the GPU is compared against this oracle for it).
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence

import numpy as np

__all__ = [
    "softmax_attention", "dual_stream", "stack_heads", "sufficient_stats", "ridge_lambda", "absorb",
    "reconstruction_error", "error_from_stats", "select_layers", "update_weight", "lse_merge",
    "biased_softmax_attention", "tempcache_match", "tempcache_merge",
]

# rows handled per numpy call; each query row is computed independently, this only bounds memory
_ROW_GROUP = 256


def softmax_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """Naive softmax attention of query rows over one key set (ISPA section 2, stage 1).

    q [n, hd], k [m, hd], v [m, hd] (any float dtype, widened to fp64).
    Returns (O [n, hd], lse [n]) with s = scale * q.k, lse = log(sum_j exp(s_j)) (natural log) and
    O = sum_j softmax(s)_j v_j.  With m == 0 there is nothing to attend to: O = 0, lse = -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n = q.shape[0]
    O = np.zeros((n, v.shape[1]), dtype=np.float64)
    lse = np.full((n,), -np.inf, dtype=np.float64)
    if k.shape[0] == 0 or n == 0:
        return O, lse
    for r0 in range(0, n, _ROW_GROUP):
        r1 = min(n, r0 + _ROW_GROUP)
        s = scale * (q[r0:r1] @ k.T)
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        l = p.sum(axis=1, keepdims=True)
        O[r0:r1] = (p @ v) / l
        lse[r0:r1] = m[:, 0] + np.log(l[:, 0])
    return O, lse


def dual_stream(q, k_sink, v_sink, k_loc, v_loc, k_hist, v_hist, scale: Optional[float] = None,
                rows: Optional[Sequence[int]] = None, with_hist: bool = True) -> Dict[str, np.ndarray]:
    """A_loc and A_full of one attention call, as separate passes (ISPA section 2, stage 1).

    Inputs are [tokens, H, hd].  `rows` optionally restricts the query rows (each row is independent).
    Returns O_loc/O_full/O_hist [n, H, hd] and lse_loc/lse_full/lse_hist [H, n].
      C1 local pass : keys = sink + current chunk
      C2 full pass  : keys = sink + current chunk + history (does not reuse C1)
      C3 hist pass  : keys = history only (exists to check the post-hoc LSE merge)
    """
    q = np.asarray(q)
    if rows is not None:
        q = q[np.asarray(rows)]
    n, H, hd = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(hd)
    out = {key: np.zeros((n, H, hd)) for key in ("O_loc", "O_full", "O_hist")}
    for key in ("lse_loc", "lse_full", "lse_hist"):
        out[key] = np.full((H, n), -np.inf)
    for h in range(H):
        kl = np.concatenate([k_sink[:, h], k_loc[:, h]], axis=0)
        vl = np.concatenate([v_sink[:, h], v_loc[:, h]], axis=0)
        kf = np.concatenate([kl, k_hist[:, h]], axis=0)
        vf = np.concatenate([vl, v_hist[:, h]], axis=0)
        out["O_loc"][:, h], out["lse_loc"][h] = softmax_attention(q[:, h], kl, vl, scale)
        out["O_full"][:, h], out["lse_full"][h] = softmax_attention(q[:, h], kf, vf, scale)
        if with_hist:
            out["O_hist"][:, h], out["lse_hist"][h] = softmax_attention(q[:, h], k_hist[:, h], v_hist[:, h], scale)
    return out


def lse_merge(O_a, lse_a, O_b, lse_b):
    """Post-hoc merge of two attention branches by their LSEs (ISPA section 2, stage 1 and
    contribution 2, "Decomposable Attention" over online-softmax state).

    O_* [n, H, hd], lse_* [H, n].  O = sigmoid(lse_a - lse_b) O_a + sigmoid(lse_b - lse_a) O_b and
    lse = logaddexp(lse_a, lse_b).  An empty branch (lse = -inf) gets weight exactly 0.
    """
    lse = np.logaddexp(lse_a, lse_b)
    with np.errstate(invalid="ignore"):
        wa = np.where(np.isneginf(lse_a), 0.0, np.exp(lse_a - lse))
        wb = np.where(np.isneginf(lse_b), 0.0, np.exp(lse_b - lse))
    O = wa.T[:, :, None] * O_a + wb.T[:, :, None] * O_b
    return O, lse


def stack_heads(O: np.ndarray) -> np.ndarray:
    """[n, H, hd] -> [n, d] with column h*hd + e: one row per query token, heads concatenated."""
    return np.asarray(O, dtype=np.float64).reshape(O.shape[0], -1)


def sufficient_stats(A_loc: np.ndarray, A_full: np.ndarray):
    """The factors of the closed form accumulated over warmup rows (ISPA section 2, stage 2).

    G = A_loc^T A_loc, R = A_loc^T (A_full - A_loc), S = D^T D with D = A_full - A_loc.
    S is not on the pages; it lets eps be evaluated from statistics alone.
    """
    A_loc = np.asarray(A_loc, dtype=np.float64)
    D = np.asarray(A_full, dtype=np.float64) - A_loc
    return A_loc.T @ A_loc, A_loc.T @ D, D.T @ D


def ridge_lambda(G: np.ndarray, lam_rel: float) -> float:
    """lam = lam_rel * trace(G) / d (the pages give no numeric lambda)."""
    return float(lam_rel) * float(np.trace(G)) / G.shape[0]


def absorb(G: np.ndarray, R: np.ndarray, W: np.ndarray, lam: float) -> np.ndarray:
    """Closed-form ridge absorb dW = (G + lam I)^-1 R W (ISPA section 2, stage 2, closed form).

    Dense LU with partial pivoting on G + lam I (LAPACK gesv), right-hand side B = R @ W.
    """
    G = np.asarray(G, dtype=np.float64)
    B = np.asarray(R, dtype=np.float64) @ np.asarray(W, dtype=np.float64)
    return np.linalg.solve(G + lam * np.eye(G.shape[0]), B)


def reconstruction_error(A_loc, A_full, W, dW):
    """Explicit data-term residual of the ridge objective at dW (ISPA section 2, objective and
    "Dynamic Layer Selection").  Returns (eps, eps_rel):
    eps = ||A_loc (W + dW) - A_full W||_F^2, eps_rel = eps / ||(A_full - A_loc) W||_F^2.
    """
    A_loc = np.asarray(A_loc, dtype=np.float64)
    A_full = np.asarray(A_full, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    E = A_loc @ (W + dW) - A_full @ W
    eps = float(np.sum(E * E))
    DW = (A_full - A_loc) @ W
    base = float(np.sum(DW * DW))
    return eps, (eps / base if base > 0 else 0.0)


def error_from_stats(G, R, S, W, dW):
    """The same residual from the statistics only (expanding the square of the objective's data term):
    eps = tr(W^T S W) - 2 tr(dW^T R W) + tr(dW^T G dW); eps_rel = eps / tr(W^T S W)."""
    W = np.asarray(W, dtype=np.float64)
    dW = np.asarray(dW, dtype=np.float64)
    sww = float(np.sum(W * (np.asarray(S, dtype=np.float64) @ W)))
    cross = float(np.sum(dW * (np.asarray(R, dtype=np.float64) @ W)))
    quad = float(np.sum(dW * (np.asarray(G, dtype=np.float64) @ dW)))
    eps = sww - 2.0 * cross + quad
    return eps, (eps / sww if sww > 0 else 0.0)


def select_layers(eps: Sequence[float], k: int) -> np.ndarray:
    """Instance-specific layer selection (ISPA section 2, "Dynamic Layer Selection"): rank all layers
    by eps ascending and return the k lowest, listed in ascending layer index.  Ties go to the lower
    layer index; NaN ranks last."""
    eps = [float(e) for e in eps]
    if k < 0 or k > len(eps):
        raise ValueError("k out of range")
    key = [(1 if math.isnan(e) else 0, 0.0 if math.isnan(e) else e, i) for i, e in enumerate(eps)]
    chosen = [t[2] for t in sorted(key)[:k]]
    return np.array(sorted(chosen), dtype=np.int32)


def update_weight(W, dW):
    """W_new = W + dW for a selected layer (ISPA section 2, stage 3)."""
    return np.asarray(W, dtype=np.float64) + np.asarray(dW, dtype=np.float64)


def project(A, W) -> np.ndarray:
    """Layer output projection y = A W in fp64 (ISPA section 2, stage 3: a layer's attention output
    times its d_in x d_out projection weight)."""
    return np.asarray(A, dtype=np.float64) @ np.asarray(W, dtype=np.float64)


def layer_forward(q, k_sink, v_sink, k_loc, v_loc, k_hist, v_hist, W, *, llayer: bool,
                  scale: Optional[float] = None, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """One layer's attention and output projection after T_warm (ISPA section 2, stage 3).

    F-Layer (llayer False): softmax attention over sink + current chunk + history, projected by W.
    L-Layer (llayer True): softmax attention over sink + current chunk only (the layer's history
    K/V are gone), projected by W (the caller passes W_new = W + dW).
    Inputs [tokens, H, hd]; W [d, d_out]; returns y [n, d_out] (fp64), one row per query token.
    """
    q = np.asarray(q)
    if rows is not None:
        q = q[np.asarray(rows)]
    n, H, hd = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(hd)
    A = np.zeros((n, H, hd))
    for h in range(H):
        parts_k = [k_sink[:, h], k_loc[:, h]] + ([] if llayer else [k_hist[:, h]])
        parts_v = [v_sink[:, h], v_loc[:, h]] + ([] if llayer else [v_hist[:, h]])
        A[:, h], _ = softmax_attention(q[:, h], np.concatenate(parts_k, axis=0), np.concatenate(parts_v, axis=0),
                                       scale)
    return project(stack_heads(A), W)


# ----------------------------------------------------------------------------- quantised projection
# NEXT row f3 (ISPA summary, section 4 / contribution list: ISPA combined with W8A8 post-training
# quantisation of the L-Layers).  The pages fix no format; the reading here is fp8 E4M3 (1 sign,
# 4 exponent bits with bias 7, 3 mantissa bits, no infinities, largest finite 448) with one fp32
# scale per activation row and one per output column of W, rounding to nearest even and
# saturating finite overflow at +-448.

E4M3_MAX = 448.0


def e4m3_round(x) -> np.ndarray:
    """Round to the nearest E4M3 value (ties to even), saturating at +-448; NaN stays NaN."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    with np.errstate(divide="ignore", invalid="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.clip(e, -6.0, 8.0)                 # binades of the normals; below 2^-6 the subnormal step
    quantum = np.exp2(e - 3.0)                 # 3 mantissa bits
    q = np.round(a / quantum) * quantum        # numpy rounds halves to even
    q = np.minimum(q, E4M3_MAX)
    return np.where(np.isnan(x), np.nan, np.copysign(q, x))


def quantize_rows(A):
    """Per-row symmetric E4M3 quantisation: s_i = max_j |A_ij| / 448 (fp32; 1 for an all-zero row),
    q_ij = e4m3(A_ij / s_i) with the division done in fp32.  Returns (q fp64 [m, n], s fp64 [m])."""
    A32 = np.asarray(A, dtype=np.float32)
    amax = np.max(np.abs(A32), axis=1)
    s = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    q = e4m3_round((A32 / s[:, None]).astype(np.float32))
    return q, s.astype(np.float64)


def quantize_cols(W):
    """Per-output-column symmetric E4M3 quantisation of W [d_in, d_out] (the same rule as
    quantize_rows applied to W^T).  Returns (q [d_in, d_out], s [d_out])."""
    q, s = quantize_rows(np.asarray(W, dtype=np.float32).T)
    return q.T, s


def project_w8a8(A, W) -> np.ndarray:
    """y = A W with both operands quantised: y_ij = s_i t_j sum_k qa_ik qw_kj (fp64 accumulation)."""
    qa, sa = quantize_rows(A)
    qw, sw = quantize_cols(W)
    return (qa @ qw) * sa[:, None] * sw[None, :]



# ----------------------------------------------------------------------------- TempCache (FAST-AR)
# NEXT row f4: the FAST-AR page ("FAST-AR", section 2 "Core components", A: TempCache) compresses the
# KV cache by merging temporally corresponding tokens: each new token finds its top-1 neighbour among
# the cached tokens, and, by the page's Lemma 5.1, merging identical keys is exact when the group's
# values are averaged and its logit is shifted by the log of the group size.  Readings of what the
# page leaves open:
#   * the neighbour is searched per head among every cached entry of that head, by cosine similarity
#     of the keys (the page names an approximate search, LSH or quantisation; the exact top-1 is its
#     limit); ties go to the lowest entry index; a zero key has similarity 0 with everything;
#   * a token merges when that similarity is >= threshold; the group keeps its first key as its
#     representative, its value becomes the mean of all members, its size grows;
#   * unmatched tokens are appended as new entries (size 1) in token order; every head keeps its own
#     entry count, entries past it have size 0;
#   * attention over the cache adds bias ln(size) to each entry's logit (-inf for size 0).

def biased_softmax_attention(q, k, v, bias, scale: float):
    """Softmax attention with a per-key logit bias: s_j = scale q.k_j + bias_j (natural-log units,
    -inf excludes key j).  q [n, hd], k/v [m, hd], bias [m].  Returns (O [n, hd], lse [n])."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    bias = np.asarray(bias, dtype=np.float64)
    n = q.shape[0]
    O = np.zeros((n, v.shape[1]))
    lse = np.full((n,), -np.inf)
    live = np.isfinite(bias) | (bias > 0)
    if not live.any() or n == 0:
        return O, lse
    s = scale * (q @ k[live].T) + bias[live][None, :]
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=1, keepdims=True)
    return (p @ v[live]) / l, m[:, 0] + np.log(l[:, 0])


def tempcache_match(k_new, k_cache, count):
    """Top-1 cached entry of every new token, per head, by cosine similarity of the keys.

    k_new [T, H, hd], k_cache [N, H, hd], count [H, N] (entries with count 0 are not candidates).
    Returns (idx int64 [H, T], sim fp64 [H, T]); idx -1 and sim -inf when a head has no entry."""
    k_new = np.asarray(k_new, dtype=np.float64)
    k_cache = np.asarray(k_cache, dtype=np.float64)
    T, H, _ = k_new.shape
    idx = np.full((H, T), -1, dtype=np.int64)
    sim = np.full((H, T), -np.inf)
    for h in range(H):
        valid = np.nonzero(np.asarray(count)[h] > 0)[0]
        if valid.size == 0:
            continue
        a = k_new[:, h]
        b = k_cache[valid, h]
        na = np.linalg.norm(a, axis=1)
        nb = np.linalg.norm(b, axis=1)
        dots = a @ b.T
        with np.errstate(divide="ignore", invalid="ignore"):
            cos = np.where((na[:, None] > 0) & (nb[None, :] > 0), dots / (na[:, None] * nb[None, :]), 0.0)
        best = np.argmax(cos, axis=1)             # first maximum: ties to the lowest entry index
        idx[h] = valid[best]
        sim[h] = cos[np.arange(T), best]
    return idx, sim


def tempcache_merge(k_cache, v_cache, count, k_new, v_new, idx, sim, threshold: float):
    """Merge one new frame into the cache (FAST-AR TempCache, Lemma 5.1), per head.

    k_cache/v_cache [N, H, hd] with count [H, N] (the first n_h entries of head h have count >= 1);
    k_new/v_new [T, H, hd]; idx/sim [H, T] from tempcache_match.  Token t of head h joins entry
    idx[h, t] when sim[h, t] >= threshold: that entry's value becomes the mean of its members
    (old mean weighted by the old count), its key is kept.  The other tokens are appended, in token
    order, after the head's last entry.  Returns (k, v, count) with N + T entries (fp64, count int64)."""
    k_cache = np.asarray(k_cache, dtype=np.float64)
    v_cache = np.asarray(v_cache, dtype=np.float64)
    count = np.asarray(count, dtype=np.int64)
    k_new = np.asarray(k_new, dtype=np.float64)
    v_new = np.asarray(v_new, dtype=np.float64)
    N, H, hd = k_cache.shape
    T = k_new.shape[0]
    k_out = np.zeros((N + T, H, hd))
    v_out = np.zeros((N + T, H, hd))
    c_out = np.zeros((H, N + T), dtype=np.int64)
    k_out[:N], v_out[:N], c_out[:, :N] = k_cache, v_cache, count
    for h in range(H):
        n_h = int(np.count_nonzero(count[h] > 0))
        sums = v_cache[:, h] * count[h][:, None]   # member sums of the existing groups
        for t in range(T):
            e = int(idx[h, t])
            if e >= 0 and sim[h, t] >= threshold:
                sums[e] += v_new[t, h]
                c_out[h, e] += 1
            else:
                k_out[n_h, h], v_out[n_h, h], c_out[h, n_h] = k_new[t, h], v_new[t, h], 1
                n_h += 1
        grown = (c_out[h, :N] > count[h]) & (count[h] > 0)
        v_out[:N, h][grown] = sums[grown] / c_out[h, :N][grown][:, None]
    return k_out, v_out, c_out
