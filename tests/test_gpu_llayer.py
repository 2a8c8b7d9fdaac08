"""GPU parity of the post-warmup layer path (ISPA section 2, stage 3): the output projection
(ispa_project) and the L-Layer / F-Layer forward against the fp64 oracle, through the C ABI.

Tolerances: bf16 operands are read exactly by both sides and the products accumulate in fp32; Y is
rounded to bf16 once (relative error <= 2^-9 per element), so the projection is held to 5e-3 relative
Frobenius error.  The layer forward adds the attention's bf16 rounding: 1e-2, as for attention.
"""
import math

import numpy as np
import pytest

import ispa_inputs as inp
from gpu_helpers import dev, host, rel
from oracle import ispa_oracle as orc

pytestmark = pytest.mark.gpu


def _bf16(x):
    return inp.round_bf16(np.asarray(x, dtype=np.float32))


@pytest.mark.parametrize("w_transposed", [False, True])
@pytest.mark.parametrize("m,d_in,d_out", [(300, 192, 256), (128, 64, 128), (1, 128, 384)])
def test_project_bf16_matches_oracle(cuda_ok, w_transposed, m, d_in, d_out):
    import torch
    from kv_cache_compression_tma_b200 import ispa
    A = _bf16(inp.gaussian((m, d_in), 21, 1))
    W = _bf16(inp.gaussian((d_in, d_out), 21, 2, 1.0 / math.sqrt(d_in)))
    Wst = np.ascontiguousarray(W.T) if w_transposed else W
    y = ispa.project(dev(A, torch.bfloat16), dev(Wst, torch.bfloat16), w_transposed=w_transposed)
    torch.cuda.synchronize()
    assert ispa.get_device_status() == 0
    assert rel(host(y), orc.project(A, W)) <= 5e-3


def test_project_full_size_sampled_rows(cuda_ok):
    """The 1.3B-like layer's shape (4680 x 1536 by 1536 x 1536), checked on sampled rows."""
    import torch
    from kv_cache_compression_tma_b200 import ispa
    m, d = 4680, 1536
    A = _bf16(inp.gaussian((m, d), 22, 1))
    W = _bf16(inp.gaussian((d, d), 22, 2, 1.0 / math.sqrt(d)))
    y = host(ispa.project(dev(A, torch.bfloat16), dev(W, torch.bfloat16)))
    rows = inp.sample_rows(m, 96, 22)
    assert rel(y[rows], orc.project(A[rows], W)) <= 5e-3
    assert rel(y[-8:], orc.project(A[-8:], W)) <= 5e-3  # the ragged last tile


def test_project_f32_matches_oracle(cuda_ok):
    import torch
    from kv_cache_compression_tma_b200 import ispa
    A = inp.gaussian((77, 40), 23, 1).astype(np.float32)
    W = inp.gaussian((40, 24), 23, 2).astype(np.float32)
    y = ispa.project(dev(A, torch.float32), dev(W, torch.float32))
    assert rel(host(y), orc.project(A, W)) <= 1e-6


def test_project_bf16_unsupported_shape_is_refused(cuda_ok):
    import torch
    from kv_cache_compression_tma_b200 import ispa
    A = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((64, 100), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ispa.IspaError) as e:
        ispa.project(A, W)
    assert e.value.status == 2


@pytest.mark.parametrize("llayer", [False, True])
def test_layer_forward_matches_oracle(cuda_ok, llayer):
    """One 1.3B-like layer at T_warm (9 frames of history): F-Layer with W, L-Layer with a second
    weight standing in for W_new; compared on sampled query rows."""
    import torch
    from kv_cache_compression_tma_b200 import llayer as ll
    wl = inp.WORKLOADS["l1_3b"]
    x = inp.attention_inputs(wl, 0, 0, seed=5)
    W = inp.weight(wl, 0, 5)
    Wn = _bf16(W + inp.gaussian(W.shape, 5, 9, 0.1 / math.sqrt(wl.d)))
    Wuse = Wn if llayer else W
    t = {k: dev(x[k], torch.bfloat16) for k in ("q", "k_sink", "v_sink", "k_loc", "v_loc", "k_hist", "v_hist")}
    y = ll.layer_forward(t["q"], t["k_sink"], t["v_sink"], t["k_loc"], t["v_loc"], t["k_hist"], t["v_hist"],
                         dev(Wuse, torch.bfloat16), llayer=llayer)
    y = host(y)
    rows = np.concatenate([np.arange(0, x["q"].shape[0], 97), [x["q"].shape[0] - 1]])
    ref = orc.layer_forward(x["q"], x["k_sink"], x["v_sink"], x["k_loc"], x["v_loc"], x["k_hist"], x["v_hist"],
                            Wuse, llayer=llayer, rows=rows)
    assert rel(y[rows], ref) <= 1e-2


def test_llayer_output_moves_toward_flayer_after_absorb(cuda_ok):
    """Property at full size (ridge optimality): after the absorb of the layer's own statistics, the
    L-Layer output A_loc W_new is closer to the F-Layer output A_full W than A_loc W is."""
    import torch
    from kv_cache_compression_tma_b200 import ispa
    wl = inp.WORKLOADS["l1_3b"]
    x = inp.attention_inputs(wl, 0, 0, seed=6)
    t = {k: dev(x[k], torch.bfloat16) for k in ("q", "k_sink", "v_sink", "k_loc", "v_loc", "k_hist", "v_hist")}
    o = ispa.dual_stream_attn(t["q"], t["k_sink"], t["v_sink"], t["k_loc"], t["v_loc"], t["k_hist"], t["v_hist"])
    d = wl.d
    G, R, S = (torch.empty((d, d), dtype=torch.float32, device="cuda") for _ in range(3))
    ispa.accum_stats(o["o_loc"], o["d"], G, R, S, zero=True)
    W = dev(inp.weight(wl, 0, 6), torch.bfloat16)
    res = ispa.absorb(G, R, S, W, 1e-2, lam_rel=True, write_wnew=True)
    y_f = ispa.project(o["o_full"], W).to(torch.float64)
    y_0 = ispa.project(o["o_loc"], W).to(torch.float64)
    y_l = ispa.project(o["o_loc"], res["w_new"]).to(torch.float64)
    torch.cuda.synchronize()
    assert ispa.get_device_status() == 0
    before = float(torch.linalg.norm(y_0 - y_f))
    after = float(torch.linalg.norm(y_l - y_f))
    assert after < before
