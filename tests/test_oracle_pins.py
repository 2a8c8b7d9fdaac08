"""Pins of the fp64 oracle against what the ISPA pages and the mathematics fix (CPU only).

The pages print no worked numeric example, so every pin here is an identity, a closed form, a
limit, brute force on tiny inputs or a second textbook route:

  P1  post-hoc LSE merge of the local and history branches equals full attention
      (ISPA section 2, stage 1: decomposable attention merged post-hoc);
  P2  empty history: A_full == A_loc, hence R = S = 0, dW = 0, eps = 0 (stage 1: A_full is the
      output over the whole history);
  P3  softmax closed forms: identical keys, one key, two keys;
  P4  brute force with scalar Python loops on the tiny shape (attention, row stacking, Gram);
  P5  planted linear history A_full = A_loc (I + C): dW(lam) = (G+lam I)^-1 G C W, dW -> C W and
      eps -> 0 as lam -> 0 (stage 2, objective and closed form);
  P6  normal equations (G + lam I) dW = R W (first-order optimality of the stage-2 objective);
  P7  ridge limits and monotonicity over a lam sweep;
  P8  optimality: the stage-2 objective is not lowered by random perturbations of dW;
  P9  a second route: ridge via the SVD of A_loc, and numpy lstsq at lam = 0;
  P10 eps from the statistics equals the explicit residual;
  P11 selection (section 2, "Dynamic Layer Selection") against brute force over subsets;
  P12 G and S symmetric positive semi-definite; Cholesky of G + lam I succeeds for lam > 0;
  P13 scale equivariance;
  P14 the output projection against a product worked by hand and the identity weight;
  P15 the layer forward after T_warm (stage 3): an L-Layer equals the local branch of stage 1
      projected by its weight, an F-Layer the full branch, and the two coincide with no history;
  P16 the point of the absorb for an L-Layer: with W_new = W + dW its output approaches the
      F-Layer output A_full W (exactly in the planted case as lam -> 0; never worse than W);
  P19 the ridge weight lam = lam_rel * trace(G) / d (the workloads' statement of lambda) against
      values worked by hand, including a G whose off-diagonal entries must not count;
  P20 FAST-AR TempCache, Lemma 5.1: merging identical keys (values averaged, logit shifted by the log
      of the group size) leaves attention unchanged;
  P21 TempCache with a threshold no similarity reaches: the cache is the plain concatenation, every
      group has size 1, and the biased softmax is the plain one;
  P22 TempCache matching against scalar-loop brute force (cosine similarity, ties to the lowest
      index, zero keys);
  P23 TempCache bookkeeping: sizes add up to the tokens seen and every group's value times its size is
      the sum of its members' values.
Mutation tests at the end plant one plausible mistake at a time into a copy of an oracle function
and check that some pin fails.
"""
import itertools
import math

import numpy as np
import pytest

import ispa_inputs as inp
from oracle import ispa_oracle as orc


# ----------------------------------------------------------------------------- helpers

def tiny_inputs(chunk=0):
    wl = inp.WORKLOADS["tiny"]
    return wl, inp.attention_inputs(wl, 0, chunk, seed=0)


def tiny_rows():
    """A_loc / A_full of the two tiny warmup chunks, stacked (M = 64 rows, d = 64)."""
    wl = inp.WORKLOADS["tiny"]
    tl = (inp.kv_timeline(wl, 0, "k"), inp.kv_timeline(wl, 0, "v"))
    Al, Af = [], []
    for c in range(len(wl.chunks)):
        x = inp.attention_inputs(wl, 0, c, seed=0, timelines=tl)
        o = orc.dual_stream(x["q"], x["k_sink"], x["v_sink"], x["k_loc"], x["v_loc"], x["k_hist"], x["v_hist"])
        Al.append(orc.stack_heads(o["O_loc"]))
        Af.append(orc.stack_heads(o["O_full"]))
    return wl, np.concatenate(Al), np.concatenate(Af)


def rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (nb if nb > 0 else 1.0)


def objective(A_loc, A_full, W, dW, lam):
    E = A_loc @ (W + dW) - A_full @ W
    return float(np.sum(E * E) + lam * np.sum(dW * dW))


def planted(M=96, d=24, seed=3):
    A = inp.gaussian((M, d), seed, 1)
    C = inp.gaussian((d, d), seed, 2, 0.3)
    W = inp.gaussian((d, d), seed, 3, 1.0 / math.sqrt(d))
    return A, A @ (np.eye(d) + C), C, W


# ----------------------------------------------------------------------------- pin checks
# Each check takes the oracle functions it exercises, so the mutation tests can feed mutants.

def check_merge_identity(dual_stream=orc.dual_stream, lse_merge=orc.lse_merge):
    wl, x = tiny_inputs(0)
    o = dual_stream(x["q"], x["k_sink"], x["v_sink"], x["k_loc"], x["v_loc"], x["k_hist"], x["v_hist"])
    O, lse = lse_merge(o["O_loc"], o["lse_loc"], o["O_hist"], o["lse_hist"])
    return max(rel(O, o["O_full"]), float(np.max(np.abs(lse - o["lse_full"]))))


def check_brute_force(dual_stream=orc.dual_stream, stack_heads=orc.stack_heads,
                      sufficient_stats=orc.sufficient_stats, n_rows=12):
    """Scalar-loop evaluation of the definitions on the tiny shape; returns the max deviation."""
    wl, x = tiny_inputs(1)
    H, hd = wl.n_heads, wl.head_dim
    scale = 1.0 / math.sqrt(hd)
    q = x["q"][:n_rows].astype(float)
    segs_loc = [(x["k_sink"], x["v_sink"]), (x["k_loc"], x["v_loc"])]
    segs_full = segs_loc + [(x["k_hist"], x["v_hist"])]

    def brute(keys):
        O = np.zeros((n_rows, H, hd))
        L = np.zeros((H, n_rows))
        for h in range(H):
            kk = [row for K, V in keys for row in K[:, h].tolist()]
            vv = [row for K, V in keys for row in V[:, h].tolist()]
            for i in range(n_rows):
                qi = q[i, h].tolist()
                s = [scale * sum(a * b for a, b in zip(qi, kr)) for kr in kk]
                mx = max(s)
                w = [math.exp(t - mx) for t in s]
                z = sum(w)
                for e in range(hd):
                    O[i, h, e] = sum(w[j] * vv[j][e] for j in range(len(vv))) / z
                L[h, i] = mx + math.log(z)
        return O, L

    Ob_l, Lb_l = brute(segs_loc)
    Ob_f, Lb_f = brute(segs_full)
    o = dual_stream(x["q"], x["k_sink"], x["v_sink"], x["k_loc"], x["v_loc"], x["k_hist"], x["v_hist"],
                    rows=np.arange(n_rows))
    err = max(np.max(np.abs(o["O_loc"] - Ob_l)), np.max(np.abs(o["O_full"] - Ob_f)),
              np.max(np.abs(o["lse_loc"] - Lb_l)), np.max(np.abs(o["lse_full"] - Lb_f)))
    # row stacking: column h*hd + e holds head h element e
    A_l, A_f = stack_heads(o["O_loc"]), stack_heads(o["O_full"])
    for i in range(n_rows):
        for h in range(H):
            for e in range(0, hd, 7):
                err = max(err, abs(A_l[i, h * hd + e] - Ob_l[i, h, e]), abs(A_f[i, h * hd + e] - Ob_f[i, h, e]))
    # Gram entries by explicit sums
    G, R, S = sufficient_stats(A_l, A_f)
    d = H * hd
    for a in range(0, d, 5):
        for b in range(0, d, 9):
            g = sum(Ob_l[i, a // hd, a % hd] * Ob_l[i, b // hd, b % hd] for i in range(n_rows))
            r = sum(Ob_l[i, a // hd, a % hd] * (Ob_f[i, b // hd, b % hd] - Ob_l[i, b // hd, b % hd]) for i in range(n_rows))
            s = sum((Ob_f[i, a // hd, a % hd] - Ob_l[i, a // hd, a % hd]) * (Ob_f[i, b // hd, b % hd] - Ob_l[i, b // hd, b % hd]) for i in range(n_rows))
            err = max(err, abs(G[a, b] - g), abs(R[a, b] - r), abs(S[a, b] - s))
    return err


def check_planted(sufficient_stats=orc.sufficient_stats, absorb=orc.absorb,
                  reconstruction_error=orc.reconstruction_error):
    A, Af, C, W = planted()
    G, R, S = sufficient_stats(A, Af)
    d = G.shape[0]
    errs = []
    for lam in (1e-3, 1.0, 50.0):
        dW = absorb(G, R, W, lam)
        closed = np.linalg.inv(G + lam * np.eye(d)) @ G @ C @ W
        errs.append(rel(dW, closed))
    dW0 = absorb(G, R, W, 1e-10)
    errs.append(rel(dW0, C @ W))
    eps, eps_rel = reconstruction_error(A, Af, W, dW0)
    errs.append(eps_rel)
    return max(errs)


def check_normal_equations(absorb=orc.absorb, seed=5):
    wl, A_l, A_f = tiny_rows()
    G, R, S = orc.sufficient_stats(A_l, A_f)
    W = inp.weight(wl, 0).astype(np.float64)
    lam = orc.ridge_lambda(G, wl.lam_rel)
    dW = absorb(G, R, W, lam)
    RW = R @ W
    return rel((G + lam * np.eye(G.shape[0])) @ dW, RW)


def check_optimality(absorb=orc.absorb, n_trials=100):
    wl, A_l, A_f = tiny_rows()
    G, R, S = orc.sufficient_stats(A_l, A_f)
    W = inp.weight(wl, 0).astype(np.float64)
    lam = orc.ridge_lambda(G, wl.lam_rel)
    dW = absorb(G, R, W, lam)
    J0 = objective(A_l, A_f, W, dW, lam)
    worst = -np.inf
    for t in range(n_trials):
        delta = inp.gaussian(dW.shape, 17, t, 1e-4 * (1 + t % 5) * (np.linalg.norm(dW) / dW.shape[0] + 1e-12))
        for sgn in (1.0, -1.0):
            worst = max(worst, J0 - objective(A_l, A_f, W, dW + sgn * delta, lam))
    return worst  # > 0 means a perturbation lowered the objective


def check_svd_route(absorb=orc.absorb):
    A, Af, C, W = planted(M=80, d=20, seed=11)
    Af = Af + inp.gaussian(Af.shape, 11, 9, 0.05)  # not exactly planted: general D
    G, R, S = orc.sufficient_stats(A, Af)
    D = Af - A
    U, sig, Vt = np.linalg.svd(A, full_matrices=False)
    errs = []
    for lam in (1e-2, 3.0):
        dW = absorb(G, R, W, lam)
        ref = Vt.T @ np.diag(sig / (sig ** 2 + lam)) @ U.T @ D @ W
        errs.append(rel(dW, ref))
    dW0 = absorb(G, R, W, 0.0)
    errs.append(rel(dW0, np.linalg.lstsq(A, D @ W, rcond=None)[0]))
    return max(errs)


def check_eps_identity(error_from_stats=orc.error_from_stats, reconstruction_error=orc.reconstruction_error):
    wl, A_l, A_f = tiny_rows()
    G, R, S = orc.sufficient_stats(A_l, A_f)
    W = inp.weight(wl, 0).astype(np.float64)
    out = []
    for lam_rel in (1e-4, 1e-3, 1e-1):
        lam = orc.ridge_lambda(G, lam_rel)
        dW = orc.absorb(G, R, W, lam)
        e1, r1 = reconstruction_error(A_l, A_f, W, dW)
        e2, r2 = error_from_stats(G, R, S, W, dW)
        out.append(abs(e1 - e2) / abs(e1))
        out.append(abs(r1 - r2) / abs(r1))
    return max(out)


def check_selection(select_layers=orc.select_layers):
    """Returns True if select_layers agrees with brute force and the tie/NaN rules."""
    for trial in range(20):
        L = 6
        eps = inp.gaussian((L,), 23, trial) ** 2
        for k in range(0, L + 1):
            best = min(itertools.combinations(range(L), k), key=lambda c: sum(eps[list(c)]))
            if list(select_layers(list(eps), k)) != sorted(best):
                return False
    if list(select_layers([1.0, 0.5, 0.5, 2.0], 2)) != [1, 2]:
        return False
    if list(select_layers([0.2, 0.1, 0.1, 0.1], 2)) != [1, 2]:
        return False
    if list(select_layers([float("nan"), 3.0, 1.0], 2)) != [1, 2]:
        return False
    if list(select_layers([float("nan"), 3.0, 1.0], 3)) != [0, 1, 2]:
        return False
    return True


# ----------------------------------------------------------------------------- the pins

def test_p1_lse_merge_equals_full_attention():
    assert check_merge_identity() <= 1e-12


def test_p1_merge_on_l1_3b_rows():
    """The merge identity on a few rows of the 1.3B-like shape (history 9 frames)."""
    wl = inp.WORKLOADS["l1_3b"]
    x = inp.attention_inputs(wl, 0, 0)
    rows = inp.sample_rows(wl.n_q(), 4, salt=1)
    o = orc.dual_stream(x["q"][:, :2], x["k_sink"][:, :2], x["v_sink"][:, :2], x["k_loc"][:, :2],
                        x["v_loc"][:, :2], x["k_hist"][:, :2], x["v_hist"][:, :2], rows=rows)
    O, lse = orc.lse_merge(o["O_loc"], o["lse_loc"], o["O_hist"], o["lse_hist"])
    assert rel(O, o["O_full"]) <= 1e-12
    assert np.max(np.abs(lse - o["lse_full"])) <= 1e-11


def test_p2_empty_history():
    wl = inp.WORKLOADS["warm30"]
    small = inp.scaled(wl, frame_tokens=16, n_sink=16, n_heads=2, head_dim=16)
    x = inp.attention_inputs(small, 0, 0)  # chunk 0 of the warmup: no history
    assert x["k_hist"].shape[0] == 0
    o = orc.dual_stream(x["q"], x["k_sink"], x["v_sink"], x["k_loc"], x["v_loc"], x["k_hist"], x["v_hist"])
    assert np.array_equal(o["O_full"], o["O_loc"])
    assert np.all(np.isneginf(o["lse_hist"]))
    A_l, A_f = orc.stack_heads(o["O_loc"]), orc.stack_heads(o["O_full"])
    G, R, S = orc.sufficient_stats(A_l, A_f)
    assert not R.any() and not S.any()
    W = inp.weight(small, 0).astype(np.float64)
    dW = orc.absorb(G, R, W, orc.ridge_lambda(G, 1e-2))
    assert not dW.any()
    assert orc.reconstruction_error(A_l, A_f, W, dW)[0] == 0.0
    assert orc.error_from_stats(G, R, S, W, dW)[0] == 0.0


def test_p3_softmax_closed_forms():
    rng_q = inp.gaussian((5, 8), 1, 1)
    v = inp.gaussian((7, 8), 1, 2)
    k_same = np.repeat(inp.gaussian((1, 8), 1, 3), 7, axis=0)
    O, lse = orc.softmax_attention(rng_q, k_same, v, 0.5)
    assert np.allclose(O, v.mean(axis=0)[None, :], rtol=0, atol=1e-14)
    s = 0.5 * rng_q @ k_same[0]
    assert np.allclose(lse, s + math.log(7), rtol=0, atol=1e-13)
    O1, lse1 = orc.softmax_attention(rng_q, k_same[:1], v[:1], 0.5)
    assert np.allclose(O1, np.repeat(v[:1], 5, axis=0), rtol=0, atol=1e-15)
    k2 = inp.gaussian((2, 8), 1, 4)
    O2, lse2 = orc.softmax_attention(rng_q, k2, v[:2], 0.3)
    s1, s2 = 0.3 * rng_q @ k2[0], 0.3 * rng_q @ k2[1]
    sig = 1.0 / (1.0 + np.exp(-(s1 - s2)))
    assert np.allclose(O2, sig[:, None] * v[0] + (1 - sig)[:, None] * v[1], rtol=0, atol=1e-14)
    assert np.allclose(lse2, np.logaddexp(s1, s2), rtol=0, atol=1e-13)
    # no keys at all
    O0, lse0 = orc.softmax_attention(rng_q, k2[:0], v[:0], 0.3)
    assert not O0.any() and np.all(np.isneginf(lse0))


def test_p3_hand_worked_example():
    """A two-key example worked by hand (tests/golden/two_key_softmax.txt)."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "two_key_softmax.txt")
    vals = {}
    for line in open(path):
        line = line.split("#")[0].strip()
        if line:
            key, val = line.split("=")
            vals[key.strip()] = [float(t) for t in val.split()]
    q = np.array([vals["q"]])
    k = np.array([vals["k0"], vals["k1"]])
    v = np.array([vals["v0"], vals["v1"]])
    O, lse = orc.softmax_attention(q, k, v, vals["scale"][0])
    assert np.allclose(O[0], vals["O"], rtol=0, atol=1e-12)
    assert abs(lse[0] - vals["lse"][0]) <= 1e-12


def test_p4_brute_force_tiny():
    assert check_brute_force() <= 1e-12


def test_p5_planted_linear_history():
    assert check_planted() <= 1e-6


def test_p6_normal_equations():
    assert check_normal_equations() <= 1e-12


def test_p7_ridge_limits_and_monotonicity():
    wl, A_l, A_f = tiny_rows()
    G, R, S = orc.sufficient_stats(A_l, A_f)
    W = inp.weight(wl, 0).astype(np.float64)
    base = np.trace(G) / G.shape[0]
    norms, epss = [], []
    for lam_rel in 10.0 ** np.arange(-6, 4):
        lam = lam_rel * base
        dW = orc.absorb(G, R, W, lam)
        norms.append(np.linalg.norm(dW))
        epss.append(orc.reconstruction_error(A_l, A_f, W, dW)[0])
    assert all(a >= b * (1 - 1e-12) for a, b in zip(norms, norms[1:]))
    assert all(a <= b * (1 + 1e-12) for a, b in zip(epss, epss[1:]))
    RW = R @ W
    for lam_rel in (1e4, 1e6):
        lam = lam_rel * base
        gap = rel(lam * orc.absorb(G, R, W, lam), RW)
        assert gap <= 3.0 * np.linalg.norm(G, 2) / lam
    # lam -> infinity: dW -> 0, eps -> ||D W||^2 (eps_rel -> 1)
    dW = orc.absorb(G, R, W, 1e12 * base)
    assert orc.reconstruction_error(A_l, A_f, W, dW)[1] == pytest.approx(1.0, abs=1e-9)


def test_p8_optimality():
    assert check_optimality() <= 1e-12 * 1.0


def test_p9_svd_and_lstsq_routes():
    assert check_svd_route() <= 1e-9


def test_p10_eps_from_stats_matches_explicit_residual():
    assert check_eps_identity() <= 1e-10


def test_p11_selection_brute_force():
    assert check_selection()
    with pytest.raises(ValueError):
        orc.select_layers([1.0, 2.0], 3)


def test_p12_stats_symmetric_psd():
    wl, A_l, A_f = tiny_rows()
    G, R, S = orc.sufficient_stats(A_l, A_f)
    for X in (G, S):
        assert np.array_equal(X, X.T) or rel(X, X.T) <= 1e-15
        assert np.linalg.eigvalsh(X).min() >= -1e-12 * np.abs(X).max()
    np.linalg.cholesky(G + orc.ridge_lambda(G, 1e-6) * np.eye(G.shape[0]))


def test_p13_scale_equivariance():
    wl, A_l, A_f = tiny_rows()
    G, R, S = orc.sufficient_stats(A_l, A_f)
    W = inp.weight(wl, 0).astype(np.float64)
    lam = orc.ridge_lambda(G, 1e-3)
    dW = orc.absorb(G, R, W, lam)
    eps = orc.reconstruction_error(A_l, A_f, W, dW)[0]
    a = 3.0
    assert rel(orc.absorb(G, R, a * W, lam), a * dW) <= 1e-12
    assert orc.reconstruction_error(A_l, A_f, a * W, a * dW)[0] == pytest.approx(a * a * eps, rel=1e-12)
    b = 0.25
    G2, R2, S2 = orc.sufficient_stats(b * A_l, b * A_f)
    assert rel(orc.absorb(G2, R2, W, b * b * lam), dW) <= 1e-10


def test_tiny_workload_geometry():
    """The tiny case's geometry: 2 chunks x 32 queries, sink 16, local 32, history 96 keys."""
    wl = inp.WORKLOADS["tiny"]
    for c in range(2):
        x = inp.attention_inputs(wl, 0, c)
        assert x["q"].shape == (32, 2, 32)
        assert x["k_sink"].shape[0] == 16 and x["k_loc"].shape[0] == 32 and x["k_hist"].shape[0] == 96
    assert wl.rows_per_layer == 64 and wl.d == 64


# ----------------------------------------------------------------------------- mutation tests

_SOFTMAX = orc.softmax_attention


def _mut_softmax_noscale(q, k, v, scale):
    return _SOFTMAX(q, k, v, 1.0)


def _mut_lse_nomax(q, k, v, scale):
    O, lse = _SOFTMAX(q, k, v, scale)
    s = scale * (np.asarray(q, float) @ np.asarray(k, float).T) if len(k) else None
    return O, (lse - s.max(axis=1) if s is not None else lse)


def _dual_with(softmax_fn):
    def ds(*a, **kw):
        saved = orc.softmax_attention
        orc.softmax_attention = softmax_fn
        try:
            return orc.dual_stream(*a, **kw)
        finally:
            orc.softmax_attention = saved
    return ds


def test_mutation_softmax_scale_dropped_is_caught():
    assert check_brute_force(dual_stream=_dual_with(_mut_softmax_noscale), n_rows=3) > 1e-6


def test_mutation_lse_without_max_is_caught():
    assert check_merge_identity(dual_stream=_dual_with(_mut_lse_nomax)) > 1e-6


def test_mutation_head_order_is_caught():
    def bad_stack(O):
        O = np.asarray(O, dtype=np.float64)
        return O.transpose(0, 2, 1).reshape(O.shape[0], -1)
    assert check_brute_force(stack_heads=bad_stack, n_rows=3) > 1e-6


def test_mutation_delta_sign_is_caught():
    def bad_stats(A_loc, A_full):
        G, R, S = orc.sufficient_stats(A_loc, A_full)
        return G, -R, S
    assert check_planted(sufficient_stats=bad_stats) > 1e-3


def test_mutation_lambda_dropped_is_caught():
    def bad_absorb(G, R, W, lam):
        return orc.absorb(G, R, W, 0.0)
    assert check_normal_equations(absorb=bad_absorb) > 1e-6


def test_mutation_transposed_operands_are_caught():
    def bad_w(G, R, W, lam):
        return orc.absorb(G, R, W.T, lam)

    def bad_r(G, R, W, lam):
        return orc.absorb(G, R.T, W, lam)
    assert check_normal_equations(absorb=bad_w) > 1e-6
    assert check_normal_equations(absorb=bad_r) > 1e-6
    assert check_optimality(absorb=bad_r, n_trials=10) > 0


def test_mutation_eps_cross_term_sign_is_caught():
    def bad_eps(G, R, S, W, dW):
        e, r = orc.error_from_stats(G, R, S, W, -dW)
        return e, r
    assert check_eps_identity(error_from_stats=bad_eps) > 1e-6


def test_mutation_descending_selection_is_caught():
    def bad_select(eps, k):
        order = sorted(range(len(eps)), key=lambda i: -eps[i])[:k]
        return np.array(sorted(order))
    assert not check_selection(bad_select)

# ----------------------------------------------------------------------------- P19: the ridge weight

def check_ridge_lambda(ridge_lambda=orc.ridge_lambda):
    """P19: lam = lam_rel * trace(G) / d, the workloads' statement of lambda, on values worked by hand.
    Returns the largest relative error over the cases (0 for the definition)."""
    cases = [
        # G = diag(1, 2, 3, 6): trace 12, d = 4, lam_rel 1e-3 -> 1e-3 * 12 / 4 = 3e-3
        (np.diag([1.0, 2.0, 3.0, 6.0]), 1e-3, 3e-3),
        # off-diagonal entries do not enter: trace 2 + 4 = 6, d = 2, lam_rel 0.5 -> 1.5
        (np.array([[2.0, 5.0], [5.0, 4.0]]), 0.5, 1.5),
        # d = 3, trace 0.3 + 0.6 + 0.9 = 1.8, lam_rel 1e-2 -> 1e-2 * 1.8 / 3 = 6e-3
        (np.array([[0.3, -1.0, 2.0], [-1.0, 0.6, 0.0], [2.0, 0.0, 0.9]]), 1e-2, 6e-3),
    ]
    return max(abs(ridge_lambda(G, lr) - want) / want for G, lr, want in cases)


def test_p19_ridge_lambda_hand_values():
    assert check_ridge_lambda() <= 1e-15


def test_mutation_ridge_lambda_slips_are_caught():
    def d_squared(G, lam_rel):
        return float(lam_rel) * float(np.trace(G)) / G.shape[0] ** 2

    def trace_plus_identity(G, lam_rel):
        return float(lam_rel) * float(np.trace(G + np.eye(G.shape[0]))) / G.shape[0]

    def all_entries(G, lam_rel):
        return float(lam_rel) * float(np.sum(G)) / G.shape[0]

    def no_divisor(G, lam_rel):
        return float(lam_rel) * float(np.trace(G))
    for bad in (d_squared, trace_plus_identity, all_entries, no_divisor):
        assert check_ridge_lambda(bad) > 1e-3, bad.__name__


# ----------------------------------------------------------------------------- stage 3 pins

def check_project_closed_form(project=orc.project):
    """P14: a product worked by hand, and the identity weight."""
    A = np.array([[1.0, 2.0, 3.0], [4.0, 5.0, 6.0]])
    W = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]])
    want = np.array([[4.0, 5.0], [10.0, 11.0]])
    e1 = np.max(np.abs(project(A, W) - want))
    B = inp.gaussian((5, 7), 11, 1)
    e2 = np.max(np.abs(project(B, np.eye(7)) - B))
    return max(e1, e2)


def check_layer_forward(layer_forward=orc.layer_forward):
    """P15: L-Layer = stage-1 local branch projected, F-Layer = full branch projected; equal with
    an empty history."""
    wl, x = tiny_inputs(1)
    d = wl.d
    W = inp.gaussian((d, d), 12, 1, 1.0 / math.sqrt(d))
    args = (x["q"], x["k_sink"], x["v_sink"], x["k_loc"], x["v_loc"], x["k_hist"], x["v_hist"])
    o = orc.dual_stream(*args)
    e1 = rel(layer_forward(*args, W, llayer=True), orc.stack_heads(o["O_loc"]) @ W)
    e2 = rel(layer_forward(*args, W, llayer=False), orc.stack_heads(o["O_full"]) @ W)
    empty = (x["q"], x["k_sink"], x["v_sink"], x["k_loc"], x["v_loc"], x["k_hist"][:0], x["v_hist"][:0])
    e3 = rel(layer_forward(*empty, W, llayer=True), layer_forward(*empty, W, llayer=False))
    return max(e1, e2, e3)


def check_llayer_gain(update_weight=orc.update_weight):
    """P16: returns (planted residual ratio at lam -> 0, worst ratio over a lam sweep on the tiny rows),
    each ratio = ||A_loc W_new - A_full W|| / ||A_loc W - A_full W||."""
    A_loc, A_full, C, W = planted()
    G, R, _ = orc.sufficient_stats(A_loc, A_full)
    dW = orc.absorb(G, R, W, 1e-10 * np.trace(G) / G.shape[0])
    target = orc.project(A_full, W)
    base = np.linalg.norm(orc.project(A_loc, W) - target)
    planted_ratio = np.linalg.norm(orc.project(A_loc, update_weight(W, dW)) - target) / base
    wl, Al, Af = tiny_rows()
    W2 = inp.gaussian((wl.d, wl.d), 13, 1, 1.0 / math.sqrt(wl.d))
    G2, R2, _ = orc.sufficient_stats(Al, Af)
    t2 = orc.project(Af, W2)
    b2 = np.linalg.norm(orc.project(Al, W2) - t2)
    worst = 0.0
    for lam_rel in (1e-4, 1e-2, 1.0, 100.0):
        dW2 = orc.absorb(G2, R2, W2, orc.ridge_lambda(G2, lam_rel))
        worst = max(worst, np.linalg.norm(orc.project(Al, update_weight(W2, dW2)) - t2) / b2)
    return planted_ratio, worst


def test_p14_projection_closed_form():
    assert check_project_closed_form() == 0.0


def test_p15_layer_forward_matches_stage1_branches():
    assert check_layer_forward() < 1e-12


def test_p16_llayer_approaches_flayer():
    planted_ratio, worst = check_llayer_gain()
    assert planted_ratio < 1e-6
    assert worst <= 1.0 + 1e-12


def test_mutation_llayer_keeps_history_is_caught():
    def bad_forward(*a, llayer, **kw):
        return orc.layer_forward(*a, llayer=False, **kw)
    assert check_layer_forward(bad_forward) > 1e-6


def test_mutation_projection_row_order_is_caught():
    # W's rows taken in the wrong order (an indexing slip between d_in and the head layout)
    assert check_project_closed_form(lambda A, W: np.asarray(A, float) @ np.asarray(W, float)[::-1]) > 1e-6


def test_mutation_llayer_without_new_weight_is_caught():
    planted_ratio, _ = check_llayer_gain(update_weight=lambda W, dW: np.asarray(W, dtype=np.float64))
    assert planted_ratio > 0.5



# ----------------------------------------------------------------------------- f3: quantised projection

def _e4m3_values():
    """Every finite E4M3 value from the bit layout (sign, 4-bit exponent with bias 7, 3-bit
    mantissa; exponent 15 with mantissa 7 is NaN)."""
    vals = []
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue
            v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
            vals += [v, -v]
    return np.unique(np.array(vals))


def test_p17_e4m3_grid_fixed_points_and_range():
    v = _e4m3_values()
    assert v.max() == 448.0 and v[v > 0].min() == 2.0 ** -9
    assert np.array_equal(orc.e4m3_round(v), v)                      # representable values are kept
    assert orc.e4m3_round(1e6) == 448.0 and orc.e4m3_round(-1e6) == -448.0   # saturation
    assert orc.e4m3_round(464.0) == 448.0                            # past the top: saturate, not NaN
    assert np.isnan(orc.e4m3_round(np.nan))


def test_p17_e4m3_ties_to_even_and_monotone():
    v = _e4m3_values()
    pos = v[v >= 0]
    mids = (pos[:-1] + pos[1:]) / 2
    got = orc.e4m3_round(mids)
    # the even neighbour is the one whose mantissa bit 0 is clear
    def mant_lsb(x):
        x = np.asarray(x)
        e = np.clip(np.floor(np.log2(np.where(x > 0, x, 1.0))), -6, 8)
        return (np.round(x / np.exp2(e - 3)).astype(np.int64)) & 1
    assert np.all((got == pos[:-1]) | (got == pos[1:]))
    assert np.all(mant_lsb(got[got > 0]) == 0)
    x = np.sort(np.random.default_rng(1).standard_normal(5000) * 50)
    assert np.all(np.diff(orc.e4m3_round(x)) >= 0)


def test_p17_e4m3_matches_torch_cast_in_range():
    import torch
    x = (np.random.default_rng(2).standard_normal(20000) * 40).astype(np.float32)
    x = x[np.abs(x) < 460]
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float32).numpy().astype(np.float64)
    assert np.array_equal(orc.e4m3_round(x), want)


def test_p18_w8a8_projection_scales_and_error():
    A = inp.gaussian((64, 96), 31, 1).astype(np.float32)
    W = inp.gaussian((96, 48), 31, 2, 0.1).astype(np.float32)
    qa, sa = orc.quantize_rows(A)
    qw, sw = orc.quantize_cols(W)
    assert np.allclose(np.max(np.abs(qa), axis=1), 448.0)           # each row's absmax lands on 448
    assert np.allclose(np.max(np.abs(qw), axis=0), 448.0)
    # elementwise dequantisation error within half an E4M3 step (relative 2^-4, plus the subnormal floor)
    assert np.all(np.abs(qa * sa[:, None] - A) <= np.abs(A) * 2.0 ** -4 + sa[:, None] * 2.0 ** -10 + 1e-12)
    y = orc.project_w8a8(A, W)
    ref = orc.project(A, W)
    err = rel(y, ref)
    assert 1e-3 < err < 0.06                                          # fp8 error, not zero, not garbage
    # an all-zero row quantises to zeros with scale 1
    q0, s0 = orc.quantize_rows(np.zeros((2, 5), np.float32))
    assert not q0.any() and np.all(s0 == 1.0)


def test_mutation_e4m3_round_half_up_is_caught():
    def bad(x):
        x = np.asarray(x, dtype=np.float64)
        a = np.abs(x)
        e = np.clip(np.floor(np.log2(np.where(a > 0, a, 1.0))), -6, 8)
        qn = np.exp2(e - 3)
        return np.copysign(np.minimum(np.floor(a / qn + 0.5) * qn, 448.0), x)
    v = _e4m3_values()
    pos = v[v >= 0]
    mids = (pos[:-1] + pos[1:]) / 2
    assert not np.array_equal(bad(mids), orc.e4m3_round(mids))


# ----------------------------------------------------------------------------- P20-P23: TempCache (FAST-AR)

def _tc_cache(seed, T=24, H=2, hd=8, dup_frac=0.5):
    """Frame 1 of T tokens (the cache), and frame 2 whose first dup_frac of tokens repeat frame 1's keys
    exactly (in a shuffled order) with fresh values; the rest are fresh keys."""
    k1 = inp.gaussian((T, H, hd), seed, 1)
    v1 = inp.gaussian((T, H, hd), seed, 2)
    perm = np.argsort(inp.gaussian((T,), seed, 3))
    k2 = inp.gaussian((T, H, hd), seed, 4)
    n_dup = int(dup_frac * T)
    k2[:n_dup] = k1[perm[:n_dup]]
    v2 = inp.gaussian((T, H, hd), seed, 5)
    return k1, v1, k2, v2, n_dup


def check_tempcache_lemma(tempcache_merge=orc.tempcache_merge, biased=orc.biased_softmax_attention, seed=61):
    """P20: attention of fresh queries over the merged cache with bias ln(size) equals attention over
    the two frames unmerged.  Returns the largest relative error over heads."""
    k1, v1, k2, v2, n_dup = _tc_cache(seed)
    T, H, hd = k1.shape
    count = np.ones((H, T), dtype=np.int64)
    idx, sim = orc.tempcache_match(k2, k1, count)
    k, v, c = tempcache_merge(k1, v1, count, k2, v2, idx, sim, 1.0 - 1e-9)
    q = inp.gaussian((5, H, hd), seed, 6)
    worst = 0.0
    for h in range(H):
        with np.errstate(divide="ignore"):
            bias = np.log(c[h].astype(np.float64))
        o_m, lse_m = biased(q[:, h], k[:, h], v[:, h], bias, 1.0 / math.sqrt(hd))
        kf = np.concatenate([k1[:, h], k2[:, h]])
        vf = np.concatenate([v1[:, h], v2[:, h]])
        o_f, lse_f = orc.softmax_attention(q[:, h], kf, vf, 1.0 / math.sqrt(hd))
        worst = max(worst, rel(o_m, o_f), float(np.max(np.abs(lse_m - lse_f))))
    return worst


def test_p20_tempcache_merging_identical_keys_is_exact():
    assert check_tempcache_lemma() <= 1e-12
    # and the merge really happened: the duplicated keys joined groups, the cache grew by the rest
    k1, v1, k2, v2, n_dup = _tc_cache(61)
    T, H, _ = k1.shape
    idx, sim = orc.tempcache_match(k2, k1, np.ones((H, T), np.int64))
    _, _, c = orc.tempcache_merge(k1, v1, np.ones((H, T), np.int64), k2, v2, idx, sim, 1.0 - 1e-9)
    for h in range(H):
        assert np.count_nonzero(c[h]) == 2 * T - n_dup
        assert np.count_nonzero(c[h] == 2) == n_dup


def test_p21_tempcache_without_merges_is_concatenation():
    k1, v1, k2, v2, _ = _tc_cache(62)
    T, H, hd = k1.shape
    count = np.ones((H, T), dtype=np.int64)
    idx, sim = orc.tempcache_match(k2, k1, count)
    k, v, c = orc.tempcache_merge(k1, v1, count, k2, v2, idx, sim, 1.5)   # cosine never exceeds 1
    assert np.array_equal(k, np.concatenate([k1, k2])) and np.array_equal(v, np.concatenate([v1, v2]))
    assert np.all(c == 1)
    q = inp.gaussian((4, H, hd), 62, 9)
    for h in range(H):
        o_b, l_b = orc.biased_softmax_attention(q[:, h], k[:, h], v[:, h], np.zeros(2 * T), 0.3)
        o_p, l_p = orc.softmax_attention(q[:, h], k[:, h], v[:, h], 0.3)
        assert rel(o_b, o_p) <= 1e-14 and np.max(np.abs(l_b - l_p)) <= 1e-13
    # -inf bias excludes a key entirely
    o_x, _ = orc.biased_softmax_attention(q[:, 0], k[:, 0], v[:, 0], np.r_[np.zeros(2 * T - 1), -np.inf], 0.3)
    o_y, _ = orc.softmax_attention(q[:, 0], k[:-1, 0], v[:-1, 0], 0.3)
    assert rel(o_x, o_y) <= 1e-14


def check_tempcache_match_brute(tempcache_match=orc.tempcache_match, seed=63):
    """P22: scalar-loop cosine similarity and argmax (first maximum), zero keys, empty entries.
    Returns the number of mismatches."""
    T, N, H, hd = 7, 9, 2, 5
    kn = inp.gaussian((T, H, hd), seed, 1)
    kc = inp.gaussian((N, H, hd), seed, 2) * np.linspace(0.2, 3.0, N)[:, None, None]  # different norms
    kc[4] = kc[2]                  # duplicate entry: a tie, resolved to the lower index 2
    kn[3] = kc[2] * 5.0            # parallel to entries 2 and 4
    kn[5] = 0.0                    # zero key: similarity 0 everywhere, first valid entry wins
    count = np.ones((H, N), dtype=np.int64)
    count[1, 0] = 0                # entry 0 of head 1 is empty
    idx, sim = tempcache_match(kn, kc, count)
    bad = 0
    for h in range(H):
        for t in range(T):
            best, best_e = -np.inf, -1
            na = math.sqrt(sum(x * x for x in kn[t, h]))
            for e in range(N):
                if count[h, e] <= 0:
                    continue
                nb = math.sqrt(sum(x * x for x in kc[e, h]))
                dot = sum(a * b for a, b in zip(kn[t, h], kc[e, h]))
                c = dot / (na * nb) if na > 0 and nb > 0 else 0.0
                if c > best + 1e-12:
                    best, best_e = c, e
            bad += int(idx[h, t] != best_e) + int(abs(sim[h, t] - best) > 1e-12)
    return bad


def test_p22_tempcache_match_brute_force():
    assert check_tempcache_match_brute() == 0


def test_p23_tempcache_bookkeeping():
    k1, v1, k2, v2, n_dup = _tc_cache(64, dup_frac=0.75)
    T, H, hd = k1.shape
    count = np.ones((H, T), dtype=np.int64)
    count[1, T - 3:] = 0           # head 1 holds fewer entries: padding after its last one
    k1[T - 3:, 1] = 0.0
    v1[T - 3:, 1] = 0.0
    idx, sim = orc.tempcache_match(k2, k1, count)
    theta = 0.2
    k, v, c = orc.tempcache_merge(k1, v1, count, k2, v2, idx, sim, theta)
    for h in range(H):
        assert c[h].sum() == count[h].sum() + T
        members = {e: [v1[e, h]] * int(count[h, e]) for e in range(T) if count[h, e] > 0}
        appended = []
        for t in range(T):
            if sim[h, t] >= theta:
                members[int(idx[h, t])].append(v2[t, h])
            else:
                appended.append(t)
        for e, vs in members.items():
            assert c[h, e] == len(vs)
            assert np.allclose(v[e, h] * c[h, e], np.sum(vs, axis=0), rtol=0, atol=1e-12)
        n_h = int(count[h].sum())
        for j, t in enumerate(appended):       # appended in token order right after the last entry
            assert c[h, n_h + j] == 1 and np.array_equal(k[n_h + j, h], k2[t, h])
        assert np.all(c[h, n_h + len(appended):] == 0)


def test_mutation_tempcache_without_log_size_bias_is_caught():
    def no_bias(q, k, v, bias, scale):
        return orc.biased_softmax_attention(q, k, v, np.where(np.isfinite(bias), 0.0, bias), scale)
    assert check_tempcache_lemma(biased=no_bias) > 1e-3


def test_mutation_tempcache_sum_instead_of_mean_is_caught():
    def summed(k_cache, v_cache, count, k_new, v_new, idx, sim, threshold):
        k, v, c = orc.tempcache_merge(k_cache, v_cache, count, k_new, v_new, idx, sim, threshold)
        return k, v * np.maximum(c.T[:, :, None], 1), c
    assert check_tempcache_lemma(tempcache_merge=summed) > 1e-3


def test_mutation_tempcache_match_by_dot_product_is_caught():
    def by_dot(k_new, k_cache, count):
        idx, sim = orc.tempcache_match(k_new, k_cache, count)
        kn = np.asarray(k_new, np.float64)
        kc = np.asarray(k_cache, np.float64)
        for h in range(kn.shape[1]):
            valid = np.nonzero(np.asarray(count)[h] > 0)[0]
            d = kn[:, h] @ kc[valid, h].T
            idx[h] = valid[np.argmax(d, axis=1)]
        return idx, sim
    assert check_tempcache_match_brute(tempcache_match=by_dot) > 0


def test_mutation_tempcache_ties_to_the_higher_index_is_caught():
    def last_max(k_new, k_cache, count):
        idx, sim = orc.tempcache_match(k_new, k_cache, count)
        kn = np.asarray(k_new, np.float64)
        kc = np.asarray(k_cache, np.float64)
        for h in range(kn.shape[1]):
            valid = np.nonzero(np.asarray(count)[h] > 0)[0]
            a, b = kn[:, h], kc[valid, h]
            na, nb = np.linalg.norm(a, axis=1), np.linalg.norm(b, axis=1)
            with np.errstate(divide="ignore", invalid="ignore"):
                cos = np.where((na[:, None] > 0) & (nb[None, :] > 0), (a @ b.T) / (na[:, None] * nb[None, :]), 0.0)
            idx[h] = valid[cos.shape[1] - 1 - np.argmax(cos[:, ::-1], axis=1)]
        return idx, sim
    assert check_tempcache_match_brute(tempcache_match=last_max) > 0
