"""ispa_absorb_static, the absorb for callers that cannot allocate device memory (an engine that owns
all device memory through its own arena, a plugin host without an allocator, or a latency-critical
loop that must not allocate at T_warm): its scratch is a library-held device array, so the caller
passes no workspace.  Checked through the C ABI against ispa_absorb with a caller workspace, on two
calls in a row (the second call runs on the array the first one left behind).

Kept in a file that pytest collects last, and self-contained: it passes alone in a fresh process
and after the other tests."""
import numpy as np
import pytest

import ispa_inputs as inp
from oracle import ispa_oracle as orc

pytestmark = pytest.mark.gpu

TOL = 5e-3  # the absorb tolerance of the other GPU tests (relative, dW and eps)


def _stats(d, seed):
    A = inp.gaussian((2 * d, d), seed, 1)
    F = A @ (np.eye(d) + inp.gaussian((d, d), seed, 2, 0.3 / np.sqrt(d))) + inp.gaussian((2 * d, d), seed, 3, 0.05)
    W = inp.gaussian((d, d), seed, 4, 1.0 / np.sqrt(d))
    G, R, S = orc.sufficient_stats(A, F)
    return [np.asarray(x, dtype=np.float32) for x in (G, R, S, W)]


def _rel(a, b):
    nb = float(np.linalg.norm(b))
    return float(np.linalg.norm(a - b)) / (nb if nb > 0 else 1.0)


def _alloc_state(torch):
    torch.cuda.synchronize()
    return (torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated(), torch.cuda.memory_reserved())


def test_absorb_static_matches_absorb_on_two_calls_in_a_row():
    import torch
    from kv_cache_compression_tma_b200 import ispa
    assert torch.cuda.is_available()
    cases = [(1536, 21, 1e-2), (256, 22, 1e-3)]
    dev = [[torch.from_numpy(x).cuda() for x in _stats(d, seed)] for d, seed, _ in cases]
    outs = [(torch.empty((d, d), dtype=torch.float32, device="cuda"), torch.empty(4, dtype=torch.float64, device="cuda"))
            for d, _, _ in cases]
    # first call on this device resolves the array's address; then two calls in a row, no allocation
    ispa.absorb_static(*dev[1][:3], dev[1][3], cases[1][2], lam_rel=True, dW=outs[1][0], eps=outs[1][1])
    before = _alloc_state(torch)  # read after a synchronize, so lazy loading on the first call is excluded
    for (d, seed, lam_rel), t, (dW, eps) in zip(cases, dev, outs):
        ispa.absorb_static(*t[:3], t[3], lam_rel, lam_rel=True, dW=dW, eps=eps)
    assert _alloc_state(torch) == before
    assert ispa.get_device_status() == ispa.ISPA_OK
    for (d, seed, lam_rel), t, (dW, eps) in zip(cases, dev, outs):
        ref = ispa.absorb(*t[:3], t[3], lam_rel, lam_rel=True)
        torch.cuda.synchronize()
        assert ispa.get_device_status() == ispa.ISPA_OK
        r_dW, r_eps = ref["dW"].double().cpu().numpy(), ref["eps"].cpu().numpy()
        g_dW, g_eps = dW.double().cpu().numpy(), eps.cpu().numpy()
        assert _rel(g_dW, r_dW) <= TOL
        assert abs(g_eps[0] - r_eps[0]) <= TOL * abs(r_eps[0])
        assert abs(g_eps[1] - r_eps[1]) <= TOL * abs(r_eps[1])


def test_absorb_static_ragged_width_bf16_transposed_weight_and_wnew():
    """A width that is a multiple of 16 but not of 128 (the CUDA-core GEMM route and a ragged last
    block), a bf16 weight in the torch Linear layout, and W_new written: against ispa_absorb and,
    for dW, against the oracle's LU solve."""
    import torch
    from kv_cache_compression_tma_b200 import ispa
    d, lam_rel = 208, 1e-2
    G, R, S, W = _stats(d, 23)
    W16 = torch.from_numpy(W).to(torch.bfloat16)
    Wt = W16.t().contiguous().cuda()                       # [d_out, d_in]
    Wb = W16.double().numpy()                              # the bf16 values both sides read (d_in x d_out)
    t = [torch.from_numpy(x).cuda() for x in (G, R, S)]
    outs = []
    for _ in range(2):                                     # two calls in a row on the shared array
        o = ispa.absorb_static(*t, Wt, lam_rel, lam_rel=True, w_transposed=True, write_wnew=True)
        torch.cuda.synchronize()
        assert ispa.get_device_status() == ispa.ISPA_OK
        outs.append({k: v.double().cpu().numpy() for k, v in o.items()})
    ref = ispa.absorb(*t, Wt, lam_rel, lam_rel=True, w_transposed=True, write_wnew=True)
    torch.cuda.synchronize()
    assert ispa.get_device_status() == ispa.ISPA_OK
    r = {k: v.double().cpu().numpy() for k, v in ref.items() if k != "ws"}
    Gd, Rd = G.astype(np.float64), R.astype(np.float64)
    dW_oracle = orc.absorb(Gd, Rd, Wb, orc.ridge_lambda(Gd, lam_rel))
    for o in outs:
        assert _rel(o["dW"], r["dW"]) <= TOL
        assert _rel(o["dW"], dW_oracle) <= TOL
        assert abs(o["eps"][0] - r["eps"][0]) <= TOL * abs(r["eps"][0])
        assert abs(o["eps"][1] - r["eps"][1]) <= TOL * abs(r["eps"][1])
        # W_new in the caller's (transposed) layout, rounded to bf16: within one bf16 step of W + dW
        want = (Wb + o["dW"]).T
        assert np.max(np.abs(o["w_new"] - want)) <= 2.0 ** -8 * np.max(np.abs(want))
        assert _rel(o["w_new"], r["w_new"]) <= TOL


def test_absorb_static_rejects_width_beyond_its_array():
    import torch
    from kv_cache_compression_tma_b200 import ispa
    d = ispa.ABSORB_STATIC_MAX_D + 16
    z = torch.zeros((d, d), dtype=torch.float32, device="cuda")
    n0 = ispa.launch_count()
    with pytest.raises(ispa.IspaError) as e:
        ispa.absorb_static(z, z, z, z, 1e-2, lam_rel=True)
    assert e.value.status == ispa.ISPA_ERR_UNSUPPORTED
    assert ispa.launch_count() == n0
