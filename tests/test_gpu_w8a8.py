"""W8A8 (fp8 E4M3) projection of the L-Layers on the GPU (ISPA summary, section 4: ISPA combined with
W8A8 post-training quantisation; section 2 stage 3: an L-Layer projects with W_new) against the
oracle's quantize_rows / quantize_cols / project_w8a8, through the C ABI.

* Quantisation is integer work: the codes and the fp32 scales must equal the oracle's bit for bit.
* The projection multiplies the same codes; it differs from the oracle's fp64 sum only by fp32
  accumulation and the final bf16 rounding of Y: relative Frobenius error <= 4e-3 (the bf16 step is
  2^-8 relative, about 2^-9.6 on average).  Against the unquantised product A W the error is the fp8
  error the oracle's P18 pin bounds (between 1e-3 and 6e-2 relative)."""
import numpy as np
import pytest

import ispa_inputs as inp
from oracle import ispa_oracle as orc
from gpu_helpers import dev, host, rel

pytestmark = pytest.mark.gpu

Y_TOL = 4e-3


def codes_to_float(q):
    import torch
    return q.view(torch.float8_e4m3fn).to(torch.float64).cpu().numpy()


def activations(m, d, seed, zero_rows=()):
    A = inp.round_bf16(inp.gaussian((m, d), seed, 1).astype(np.float32) * np.float32(0.7))
    A[list(zero_rows)] = 0.0
    return A


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_quantize_rows_bit_exact(cuda_ok, dtype):
    import torch
    from kv_cache_compression_tma_b200 import ispa
    A = inp.gaussian((300, 1536), 51, 1).astype(np.float32)
    A[7] = 0.0                                       # an all-zero row: scale 1, zero codes
    A[3, 11] = 1e4                                   # one large entry: the rest of its row goes subnormal
    if dtype == "bf16":
        A = inp.round_bf16(A)
    X = dev(A, torch.bfloat16 if dtype == "bf16" else torch.float32)
    q, s = ispa.quantize_e4m3(X)
    torch.cuda.synchronize()
    qo, so = orc.quantize_rows(A)
    assert np.array_equal(s.cpu().numpy().astype(np.float64), so)
    assert np.array_equal(codes_to_float(q), qo)


def test_quantize_rows_bit_exact_many_scales(cuda_ok):
    """4096 bf16 rows with scales spread over 2^-40 .. 2^40 (values of every size relative to their
    scale, tiny ones included) must give the oracle's codes and scales bit for bit."""
    import torch
    from kv_cache_compression_tma_b200 import ispa
    rng = np.random.default_rng(52)
    A = rng.standard_normal((4096, 1536)).astype(np.float32)
    A *= np.exp2(rng.uniform(-40, 40, size=(4096, 1))).astype(np.float32)
    A[:, ::7] *= np.float32(1e-3)  # a share of small entries in every row
    A = inp.round_bf16(A)
    q, s = ispa.quantize_e4m3(dev(A, torch.bfloat16))
    torch.cuda.synchronize()
    qo, so = orc.quantize_rows(A)
    assert np.array_equal(s.cpu().numpy().astype(np.float64), so)
    assert np.array_equal(codes_to_float(q), qo)


def test_quantize_columns_transposed_bit_exact(cuda_ok):
    import torch
    from kv_cache_compression_tma_b200 import ispa
    W = inp.round_bf16(inp.gaussian((1536, 1024), 53, 2, 1.0 / np.sqrt(1536)).astype(np.float32))
    W[:, 5] = 0.0
    q, s = ispa.quantize_e4m3(dev(W, torch.bfloat16), columns=True)
    torch.cuda.synchronize()
    assert tuple(q.shape) == (1024, 1536)
    qo, so = orc.quantize_cols(W)
    assert np.array_equal(s.cpu().numpy().astype(np.float64), so)
    assert np.array_equal(codes_to_float(q), qo.T)
    # the torch Linear layout (d_out x d_in) quantised per row gives the same codes and scales
    q2, s2 = ispa.quantize_e4m3(dev(np.ascontiguousarray(W.T), torch.bfloat16))
    torch.cuda.synchronize()
    assert torch.equal(q2, q) and torch.equal(s2, s)


@pytest.mark.parametrize("m,d,n_rows", [(300, 1536, 300), (4680, 1536, 384), (4680, 5120, 192)])
def test_w8a8_projection_against_oracle(cuda_ok, m, d, n_rows):
    import torch
    from kv_cache_compression_tma_b200 import ispa
    A = activations(m, d, 54 + d)
    W = inp.round_bf16(inp.gaussian((d, d), 55 + d, 3, 1.0 / np.sqrt(d)).astype(np.float32))
    qa, sa = ispa.quantize_e4m3(dev(A, torch.bfloat16))
    qw, sw = ispa.quantize_e4m3(dev(W, torch.bfloat16), columns=True)
    Y = ispa.project_w8a8(qa, sa, qw, sw)
    torch.cuda.synchronize()
    assert ispa.get_device_status() == ispa.ISPA_OK
    rows = inp.sample_rows(m, n_rows, seed=d, salt=3)
    y = host(Y)[rows]
    ref = orc.project_w8a8(A[rows], W)               # per-row quantisation: a row subset is exact
    assert rel(y, ref) <= Y_TOL
    err_fp8 = rel(y, orc.project(A[rows], W))
    assert 1e-3 < err_fp8 < 6e-2


def test_w8a8_unsupported_shapes_are_refused(cuda_ok):
    import torch
    from kv_cache_compression_tma_b200 import ispa
    qa = torch.zeros((64, 192), dtype=torch.uint8, device="cuda")   # d_in not a multiple of 128
    sa = torch.ones(64, device="cuda")
    qw = torch.zeros((256, 192), dtype=torch.uint8, device="cuda")
    sw = torch.ones(256, device="cuda")
    with pytest.raises(ispa.IspaError) as e:
        ispa.project_w8a8(qa, sa, qw, sw)
    assert e.value.status == ispa.ISPA_ERR_UNSUPPORTED
