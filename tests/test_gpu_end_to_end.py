"""End-to-end parity of the ISPA hot path on the GPU: dual-stream attention over the warmup chunks,
statistics accumulation, absorb, reconstruction error and layer selection (ISPA summary, section 2,
stages 1-3 and "Dynamic Layer Selection")."""
import numpy as np
import pytest

import ispa_inputs as inp
from oracle import ispa_oracle as orc
from gpu_helpers import assert_attention_ok, attention_errors, dev, host, rel, run_attention, torch_dtype

pytestmark = pytest.mark.gpu


def gpu_layer(wl, layer, seed=0, rows_check=None, tl=None, keep_rows=True):
    """Runs every warmup chunk of one layer on the GPU and returns the device statistics, the
    per-chunk attention outputs (host copies of A_loc and D) and the attention errors of sampled rows."""
    import torch
    from kv_cache_compression_tma_b200 import ispa
    d = wl.d
    dt = torch_dtype(wl)
    GRS = [torch.empty((d, d), dtype=torch.float32, device="cuda") for _ in range(3)]
    if tl is None:
        tl = (inp.kv_timeline(wl, layer, "k", seed), inp.kv_timeline(wl, layer, "v", seed))
    A_loc, D, errs = [], [], []
    for c in range(len(wl.chunks)):
        x = inp.attention_inputs(wl, layer, c, seed, timelines=tl)
        out = run_attention(x, dt)
        ispa.accum_stats(out["o_loc"], out["d"], *GRS, zero=(c == 0))
        if keep_rows:
            A_loc.append(host(out["o_loc"]))
            D.append(host(out["d"]))
        if rows_check is not None:
            rows = inp.sample_rows(wl.n_q(c), rows_check, seed=seed, salt=100 * layer + c)
            ref = orc.dual_stream(x["q"], x["k_sink"], x["v_sink"], x["k_loc"], x["v_loc"], x["k_hist"], x["v_hist"],
                                  rows=rows, with_hist=True)
            errs.append(attention_errors(out, ref, rows=rows))
    torch.cuda.synchronize()
    if not keep_rows:
        return GRS, None, None, errs
    return GRS, np.concatenate(A_loc), np.concatenate(D), errs


def test_tiny_end_to_end_against_oracle(cuda_ok):
    """Tiny fp32 case, level A: every quantity against the oracle computed from the inputs alone."""
    from kv_cache_compression_tma_b200 import ispa
    wl = inp.WORKLOADS["tiny"]
    GRS, A_loc, D, errs = gpu_layer(wl, 0, rows_check=32)
    W = inp.weight(wl, 0)
    out = ispa.absorb(*GRS, dev(W, torch_dtype(wl)), wl.lam_rel, lam_rel=True, write_wnew=True)
    assert ispa.get_device_status() == 0
    # oracle, from the inputs only
    tl = (inp.kv_timeline(wl, 0, "k"), inp.kv_timeline(wl, 0, "v"))
    Al, Af = [], []
    for c in range(2):
        x = inp.attention_inputs(wl, 0, c, timelines=tl)
        o = orc.dual_stream(x["q"], x["k_sink"], x["v_sink"], x["k_loc"], x["v_loc"], x["k_hist"], x["v_hist"])
        Al.append(orc.stack_heads(o["O_loc"]))
        Af.append(orc.stack_heads(o["O_full"]))
    Al, Af = np.concatenate(Al), np.concatenate(Af)
    G, R, S = orc.sufficient_stats(Al, Af)
    lam = orc.ridge_lambda(G, wl.lam_rel)
    dW = orc.absorb(G, R, W, lam)
    eps, eps_rel = orc.reconstruction_error(Al, Af, W, dW)
    assert rel(host(GRS[0]), G) <= 1e-4 and rel(host(GRS[1]), R) <= 1e-3 and rel(host(GRS[2]), S) <= 1e-3
    assert rel(host(out["dW"]), dW) <= 5e-3
    e = host(out["eps"])
    assert abs(e[0] - eps) <= 5e-3 * eps and abs(e[1] - eps_rel) <= 5e-3 * eps_rel
    assert rel(host(out["w_new"]), orc.update_weight(W, dW)) <= 5e-3
    idx, mask, st = ispa.select_layers([e[0]], 1)
    assert list(idx) == [0]


def test_l1_3b_layer_statistics_and_absorb(cuda_ok):
    """One 1.3B-like layer and chunk: attention (sampled rows vs oracle), statistics vs an fp64 Gram of
    the GPU's own A_loc and D (level B), absorb vs the oracle LU on the GPU's statistics (level B)."""
    from kv_cache_compression_tma_b200 import ispa
    wl = inp.WORKLOADS["l1_3b"]
    GRS, A_loc, D, errs = gpu_layer(wl, 0, rows_check=64)
    for e in errs:
        assert_attention_ok(e)
    G, R, S = (host(t) for t in GRS)
    tol = A_loc.shape[0] * 2.0 ** -24  # fp32 accumulation of exact bf16 products over the chunk's rows
    assert rel(G, A_loc.T @ A_loc) <= tol and rel(R, A_loc.T @ D) <= tol and rel(S, D.T @ D) <= tol
    W = inp.weight(wl, 0)
    out = ispa.absorb(*GRS, dev(W, torch_dtype(wl)), wl.lam_rel, lam_rel=True)
    assert ispa.get_device_status() == 0
    lam = orc.ridge_lambda(G, wl.lam_rel)
    dW = orc.absorb(G, R, W, lam)
    eps_ref, eps_rel_ref = orc.error_from_stats(G, R, S, W, dW)
    e = host(out["eps"])
    assert rel(host(out["dW"]), dW) <= 5e-3
    assert abs(e[0] - eps_ref) <= 5e-3 * abs(eps_ref)
    assert abs(e[1] - eps_rel_ref) <= 5e-3 * abs(eps_rel_ref)


@pytest.mark.parametrize("n_layers", [30])
def test_warmup_selection_level_b(cuda_ok, n_layers):
    """The 1.3B-like warmup (4 chunks, history 0 -> 9 frames) on all 30 layers: eps per layer and the
    K = 15 selected layers against the oracle on the GPU's statistics."""
    from kv_cache_compression_tma_b200 import ispa
    wl = inp.WORKLOADS["warm30"]
    eps_gpu, eps_ref = [], []
    for l in range(n_layers):
        GRS, _, _, errs = gpu_layer(wl, l, rows_check=16 if l == 0 else None, keep_rows=False)
        for e in errs:
            assert_attention_ok(e)
        W = inp.weight(wl, l)
        out = ispa.absorb(*GRS, dev(W, torch_dtype(wl)), wl.lam_rel, lam_rel=True)
        assert ispa.get_device_status() == 0
        eps_gpu.append(host(out["eps"])[0])
        G, R, S = (host(t) for t in GRS)
        lam = orc.ridge_lambda(G, wl.lam_rel)
        eps_ref.append(orc.error_from_stats(G, R, S, W, orc.absorb(G, R, W, lam))[0])
    k = wl.k_select if n_layers == wl.n_layers else n_layers // 2
    idx, mask, st = ispa.select_layers(eps_gpu, k)
    ref_idx = orc.select_layers(eps_ref, k)
    srt = sorted(eps_ref)
    gap = (srt[k] - srt[k - 1]) / srt[k - 1]
    max_err = max(abs(a - b) / abs(b) for a, b in zip(eps_gpu, eps_ref))
    assert max_err <= 5e-3
    # the input recipe spreads the layers' logit scales so that the boundary gap dwarfs the numerical
    # error; a gap within twice the error would be a tie, not a pass
    assert gap > 2 * max_err, (gap, max_err)
    assert list(idx) == list(ref_idx)


def test_l14b_layer_level_b(cuda_ok):
    """One 14B-like layer (d = 5120, 40 heads) over the four warmup chunks: attention on sampled rows
    against the oracle, sampled entries of G, R, S against fp64 dot products of the GPU's own A_loc
    and D, and the 5120-wide absorb against the oracle's LU on the GPU's statistics."""
    from kv_cache_compression_tma_b200 import ispa
    wl = inp.WORKLOADS["l14b"]
    GRS, A_loc, D, errs = gpu_layer(wl, 0, rows_check=8)
    for e in errs:
        assert_attention_ok(e)
    G, R, S = (host(t) for t in GRS)
    rng = np.random.default_rng(5)
    ij = rng.integers(0, wl.d, size=(64, 2))
    tol = A_loc.shape[0] * 2.0 ** -24
    for X, (P, Q) in ((G, (A_loc, A_loc)), (R, (A_loc, D)), (S, (D, D))):
        ref = np.array([P[:, i] @ Q[:, j] for i, j in ij])
        got = np.array([X[i, j] for i, j in ij])
        scale = np.linalg.norm(ref)
        assert np.linalg.norm(got - ref) <= tol * scale + 1e-6 * scale
    W = inp.weight(wl, 0)
    out = ispa.absorb(*GRS, dev(W, torch_dtype(wl)), wl.lam_rel, lam_rel=True)
    assert ispa.get_device_status() == 0
    lam = orc.ridge_lambda(G, wl.lam_rel)
    dW = orc.absorb(G, R, W, lam)
    eps_ref, eps_rel_ref = orc.error_from_stats(G, R, S, W, dW)
    e = host(out["eps"])
    assert rel(host(out["dW"]), dW) <= 5e-3
    assert abs(e[0] - eps_ref) <= 5e-3 * abs(eps_ref)
    assert abs(e[1] - eps_rel_ref) <= 5e-3 * abs(eps_rel_ref)


def test_l14b_selection_level_b(cuda_ok):
    """The 14B-like warmup (d = 5120, 40 heads; 4 chunks, history 0 -> 9 frames) on all 40 layers:
    each layer's eps against the oracle's LU solve on the GPU's statistics (level B), and the K = 20
    selected layers identical to the oracle's (ISPA summary, section 2, "Dynamic Layer Selection").
    The oracle's 5120-wide solve of one layer runs on a worker thread while the GPU runs the next."""
    import concurrent.futures as cf
    import torch
    from kv_cache_compression_tma_b200 import ispa
    wl = inp.WORKLOADS["l14b"]

    def oracle_eps(G, R, S, W):
        lam = orc.ridge_lambda(G, wl.lam_rel)
        return orc.error_from_stats(G, R, S, W, orc.absorb(G, R, W, lam))[0]

    eps_gpu, futs = [], []
    with cf.ThreadPoolExecutor(max_workers=1) as pool:
        for l in range(wl.n_layers):
            GRS, _, _, errs = gpu_layer(wl, l, rows_check=4 if l == 0 else None, keep_rows=False)
            for e in errs:
                assert_attention_ok(e)
            W = inp.weight(wl, l)
            out = ispa.absorb(*GRS, dev(W, torch_dtype(wl)), wl.lam_rel, lam_rel=True)
            assert ispa.get_device_status() == 0
            eps_gpu.append(host(out["eps"])[0])
            G, R, S = (host(t) for t in GRS)
            del GRS, out
            torch.cuda.empty_cache()
            futs.append(pool.submit(oracle_eps, G, R, S, W))
        eps_ref = [f.result() for f in futs]
    k = wl.k_select
    idx, mask, st = ispa.select_layers(eps_gpu, k)
    ref_idx = orc.select_layers(eps_ref, k)
    srt = sorted(eps_ref)
    gap = (srt[k] - srt[k - 1]) / srt[k - 1]
    max_err = max(abs(a - b) / abs(b) for a, b in zip(eps_gpu, eps_ref))
    assert max_err <= 5e-3, max_err
    assert gap > 2 * max_err, (gap, max_err)
    assert list(idx) == list(ref_idx)
