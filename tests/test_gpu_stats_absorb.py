"""GPU parity of the warmup statistics (ISPA summary, section 2, stage 2: the factors A_loc^T A_loc
and A_loc^T (A_full - A_loc), plus D^T D) and of the closed-form ridge absorb with its
reconstruction error, through the C ABI.

Statistics are compared with an fp64 Gram of the same bf16 operands (this isolates the tensor-core
kernel: bf16 products are exact, so only fp32 accumulation order differs).  The absorb is compared
with the oracle's dense LU solve on the GPU's fp32 statistics widened to fp64 (this isolates the
solve): tolerance 5e-3 relative on dW and eps, identical selected layers."""
import numpy as np
import pytest

import ispa_inputs as inp
from oracle import ispa_oracle as orc
from gpu_helpers import dev, host, rel

pytestmark = pytest.mark.gpu


def bf16(x):
    return inp.round_bf16(np.asarray(x, dtype=np.float32))


def gram_ref(A, D):
    A = A.astype(np.float64)
    D = D.astype(np.float64)
    return A.T @ A, A.T @ D, D.T @ D


def run_stats(A, X2, dtype, second_is_full=False, zero=True, GRS=None):
    import torch
    from kv_cache_compression_tma_b200 import ispa
    d = A.shape[1]
    if GRS is None:
        GRS = [torch.empty((d, d), dtype=torch.float32, device="cuda") for _ in range(3)]
    ispa.accum_stats(dev(A, dtype), dev(X2, dtype), *GRS, second_is_full=second_is_full, zero=zero)
    torch.cuda.synchronize()
    return GRS


@pytest.mark.parametrize("m,d", [(300, 256), (64, 128), (4680, 1536)])
def test_stats_tensor_core_vs_fp64_gram(cuda_ok, m, d):
    import torch
    A = bf16(inp.gaussian((m, d), 1, m))
    D = bf16(inp.gaussian((m, d), 2, m, 0.3))
    G, R, S = (host(t) for t in run_stats(A, D, torch.bfloat16))
    Gr, Rr, Sr = gram_ref(A, D)
    # bf16 products are exact; fp32 accumulation over m rows is bounded by m * 2^-24 relative
    tol = max(1e-5, m * 2.0 ** -24)
    assert rel(G, Gr) <= tol and rel(R, Rr) <= tol and rel(S, Sr) <= tol, (rel(G, Gr), rel(R, Rr), rel(S, Sr))


def test_stats_second_input_full_and_accumulation(cuda_ok):
    """A_full given instead of D: the D products are expanded into exact bf16 products; a second call
    accumulates."""
    import torch
    m, d = 200, 256
    A = bf16(inp.gaussian((m, d), 3, 1))
    F = bf16(A + inp.gaussian((m, d), 3, 2, 0.2))
    Gr, Rr, Sr = gram_ref(A, F.astype(np.float64) - A)
    GRS = run_stats(A, F, torch.bfloat16, second_is_full=True)
    G, R, S = (host(t) for t in GRS)
    assert rel(G, Gr) <= 1e-5 and rel(R, Rr) <= 1e-4 and rel(S, Sr) <= 1e-4
    GRS = run_stats(A, F, torch.bfloat16, second_is_full=True, zero=False, GRS=GRS)
    G2, R2, S2 = (host(t) for t in GRS)
    assert rel(G2, 2 * Gr) <= 1e-5 and rel(R2, 2 * Rr) <= 1e-4 and rel(S2, 2 * Sr) <= 1e-4


def test_stats_cuda_core_fp32(cuda_ok):
    import torch
    m, d = 64, 64
    A = inp.gaussian((m, d), 4, 1).astype(np.float32)
    F = (A + inp.gaussian((m, d), 4, 2, 0.2)).astype(np.float32)
    for full in (False, True):
        second = F if full else (F.astype(np.float64) - A).astype(np.float32)
        G, R, S = (host(t) for t in run_stats(A, second, torch.float32, second_is_full=full))
        Gr, Rr, Sr = gram_ref(A, F.astype(np.float64) - A)
        assert rel(G, Gr) <= 1e-5 and rel(R, Rr) <= 1e-5 and rel(S, Sr) <= 1e-5


def run_absorb(G, R, S, W, lam, lam_rel=False, w_dtype=None, **kw):
    import torch
    from kv_cache_compression_tma_b200 import ispa
    w_dtype = w_dtype or torch.float32
    out = ispa.absorb(dev(G, torch.float32), dev(R, torch.float32), dev(S, torch.float32), dev(W, w_dtype), lam,
                      lam_rel=lam_rel, **kw)
    torch.cuda.synchronize()
    st = ispa.get_device_status()
    return out, st


def planted_stats(M, d, seed, noise=0.05):
    A = inp.gaussian((M, d), seed, 1)
    C = inp.gaussian((d, d), seed, 2, 0.3 / np.sqrt(d))
    F = A @ (np.eye(d) + C) + inp.gaussian((M, d), seed, 3, noise)
    W = inp.gaussian((d, d), seed, 4, 1.0 / np.sqrt(d))
    return (*orc.sufficient_stats(A, F), W)


def f32(x):
    return np.asarray(x, dtype=np.float32).astype(np.float64)


@pytest.mark.parametrize("d,lam_rel", [(64, 1e-3), (256, 1e-2), (384, 1e-4), (1536, 1e-2), (3072, 1e-2),
                                       (3200, 1e-2)])
def test_absorb_vs_oracle_lu(cuda_ok, d, lam_rel):
    """d = 3072 and 3200: the two-level schedule of wide layers; at 3072 the large products (B = R W
    and the substitution updates) run on 128 x 256 GEMM tiles, at 3200 a last outer block of one 128
    block and 128-wide tiles only."""
    G, R, S, W = planted_stats(max(2 * d, 256), d, seed=d)
    G, R, S, W = f32(G), f32(R), f32(S), f32(W)  # both sides read the same fp32 values
    out, st = run_absorb(G, R, S, W, lam_rel, lam_rel=True)
    assert st == 0
    lam = orc.ridge_lambda(G, lam_rel)
    dW_ref = orc.absorb(G, R, W, lam)
    eps_ref, eps_rel_ref = orc.error_from_stats(G, R, S, W, dW_ref)
    eps = host(out["eps"])
    assert abs(eps[2] - lam) <= 1e-6 * lam
    assert rel(host(out["dW"]), dW_ref) <= 5e-3
    if lam_rel == 1e-2:
        # the split-tf32 products keep the solve near fp32 accuracy on these well-conditioned
        # systems (measured 0.5-3.2e-5 at d = 256-3072); a product that dropped to tf32 accuracy
        # (a lost lo term, or a tensor core rounding instead of truncating an fp32 operand to tf32)
        # would raise it by an order of magnitude
        assert rel(host(out["dW"]), dW_ref) <= 2e-4
    assert abs(eps[0] - eps_ref) <= 5e-3 * abs(eps_ref)
    assert abs(eps[1] - eps_rel_ref) <= 5e-3 * abs(eps_rel_ref)
    # normal equations on the GPU's result
    dW = host(out["dW"])
    assert rel((G + lam * np.eye(d)) @ dW, R @ W) <= 1e-3


@pytest.mark.parametrize("d", [256, 3072])
def test_absorb_bf16_weight_transposed_and_wnew(cuda_ok, d):
    """A bf16 weight (exact in tf32: its products skip the split of W), in the torch Linear layout;
    d = 3072 runs the two-level schedule."""
    import torch
    G, R, S, W = planted_stats(2 * d, d, seed=9)
    G, R, S = f32(G), f32(R), f32(S)
    Wb = bf16(W).astype(np.float64)           # d_in x d_out
    out, st = run_absorb(G, R, S, Wb.T.copy(), 0.05, w_dtype=torch.bfloat16, w_transposed=True, write_wnew=True)
    assert st == 0
    dW_ref = orc.absorb(G, R, Wb, 0.05)
    assert rel(host(out["dW"]), dW_ref) <= 5e-3
    wn = host(out["w_new"])                   # same (transposed) orientation as the W given
    assert rel(wn, orc.update_weight(Wb, dW_ref).T) <= 5e-3


def test_absorb_no_history_gives_zero(cuda_ok):
    d = 128
    A = inp.gaussian((256, d), 11, 1)
    G = A.T @ A
    Z = np.zeros((d, d))
    W = inp.gaussian((d, d), 11, 2, 1 / np.sqrt(d))
    out, st = run_absorb(f32(G), Z, Z, f32(W), 1e-2, lam_rel=True)
    assert st == 0
    assert not host(out["dW"]).any()
    assert host(out["eps"])[0] == 0.0


def test_absorb_not_spd_sets_status(cuda_ok):
    """A negative-definite system (chosen on the host) is reported through the status word; the
    kernel neither traps nor hangs."""
    d = 128
    G = -np.eye(d)
    W = np.eye(d)
    out, st = run_absorb(G, np.eye(d), np.eye(d), W, 0.0)
    from kv_cache_compression_tma_b200 import ispa
    assert st == ispa.ISPA_ERR_NOT_SPD
    assert ispa.get_device_status() == ispa.ISPA_OK  # cleared by the previous read


def test_absorb_selection_over_layers(cuda_ok):
    """eps of several layers from GPU absorbs, ranked on the host, equals the oracle's selection on
    the same statistics."""
    from kv_cache_compression_tma_b200 import ispa
    d, L = 128, 8
    eps_gpu, eps_ref = [], []
    for l in range(L):
        G, R, S, W = planted_stats(256, d, seed=100 + l, noise=0.02 * (1 + l))
        G, R, S, W = f32(G), f32(R), f32(S), f32(W)
        out, st = run_absorb(G, R, S, W, 1e-2, lam_rel=True)
        assert st == 0
        eps_gpu.append(host(out["eps"])[0])
        lam = orc.ridge_lambda(G, 1e-2)
        eps_ref.append(orc.error_from_stats(G, R, S, W, orc.absorb(G, R, W, lam))[0])
    idx, mask, st = ispa.select_layers(eps_gpu, L // 2)
    assert list(idx) == list(orc.select_layers(eps_ref, L // 2))
    assert max(abs(a - b) / abs(b) for a, b in zip(eps_gpu, eps_ref)) <= 5e-3
