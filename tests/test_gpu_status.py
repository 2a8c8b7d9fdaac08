"""The device-status path on the GPU, exercised without faulting or hanging it.

* A bounded wait that runs out: with the test hook ISPA_TEST_ATTN_NO_LOADS the attention kernel's
  TMA producer issues nothing, so nothing is ever in flight; every consumer gives up after its
  bounded wait (about 1 s), the CTA releases its tensor memory and returns, and the status word
  reports ISPA_ERR_TIMEOUT.  The next call on the same device, hook off, must pass parity again.
* Non-finite inputs planted on the host: a NaN in the weight makes dW and eps non-finite
  (ISPA_ERR_NONFINITE); a NaN on the diagonal of G makes a Cholesky pivot non-finite
  (ISPA_ERR_NOT_SPD).  Control flow never depends on the values, so neither can hang.
"""
import time

import numpy as np
import pytest

import ispa_inputs as inp
from oracle import ispa_oracle as orc
from gpu_helpers import assert_attention_ok, attention_errors, dev, host, run_attention, torch_dtype

pytestmark = pytest.mark.gpu


def small():
    return inp.Workload("status", 2, 128, 100, 40, 3, inp._single_chunk(3, 3), 1, None, 1e-2, 0.9, 2.0, "bf16")


def _oracle(x):
    ref = orc.dual_stream(x["q"], x["k_sink"], x["v_sink"], x["k_loc"], x["v_loc"], x["k_hist"], x["v_hist"])
    ref["with_hist"] = True
    return ref


def test_bounded_wait_runs_out_and_the_next_call_recovers(cuda_ok):
    import torch
    from kv_cache_compression_tma_b200 import ispa
    wl = small()
    x = inp.attention_inputs(wl, 0, 0, seed=8)
    assert ispa.get_device_status() == ispa.ISPA_OK
    ispa.test_set_flags(ispa.ISPA_TEST_ATTN_NO_LOADS)
    try:
        t0 = time.perf_counter()
        run_attention(x, torch_dtype(wl))          # launches, then synchronises
        waited = time.perf_counter() - t0
    finally:
        ispa.test_set_flags(0)
    assert ispa.get_device_status() == ispa.ISPA_ERR_TIMEOUT
    assert 0.5 < waited < 30.0                      # the bounded wait (about 1 s), not a hang
    assert ispa.get_device_status() == ispa.ISPA_OK  # the read cleared the word
    # the context is still usable: the same call with the hook off passes parity
    out = run_attention(x, torch_dtype(wl))
    assert ispa.get_device_status() == ispa.ISPA_OK
    assert_attention_ok(attention_errors(out, _oracle(x)))
    torch.cuda.synchronize()


def test_test_hook_rejects_unknown_bits(cuda_ok):
    from kv_cache_compression_tma_b200 import ispa
    with pytest.raises(ispa.IspaError) as e:
        ispa.test_set_flags(0x80)
    assert e.value.status == ispa.ISPA_ERR_INVALID_ARG


def _stats(d, seed):
    A = inp.gaussian((2 * d, d), seed, 1)
    F = A + inp.gaussian((2 * d, d), seed, 2, 0.1)
    G, R, S = orc.sufficient_stats(A, F)
    W = inp.gaussian((d, d), seed, 3, 1.0 / np.sqrt(d))
    return [np.asarray(t, np.float32) for t in (G, R, S, W)]


def test_nan_in_weight_reports_nonfinite(cuda_ok):
    import torch
    from kv_cache_compression_tma_b200 import ispa
    G, R, S, W = _stats(256, 41)
    W[17, 3] = np.nan
    out = ispa.absorb(*(dev(t, torch.float32) for t in (G, R, S)), dev(W, torch.float32), 1e-2, lam_rel=True)
    assert ispa.get_device_status() == ispa.ISPA_ERR_NONFINITE
    assert not np.isfinite(host(out["eps"])[0])
    # and a clean call afterwards is clean again
    W[17, 3] = 0.0
    out = ispa.absorb(*(dev(t, torch.float32) for t in (G, R, S)), dev(W, torch.float32), 1e-2, lam_rel=True)
    assert ispa.get_device_status() == ispa.ISPA_OK
    assert np.isfinite(host(out["eps"])).all()


@pytest.mark.parametrize("d", [256, 1536])
def test_nan_on_the_diagonal_of_g_reports_not_spd(cuda_ok, d):
    import torch
    from kv_cache_compression_tma_b200 import ispa
    G, R, S, W = _stats(d, 42)
    G[d // 2, d // 2] = np.nan
    ispa.absorb(*(dev(t, torch.float32) for t in (G, R, S)), dev(W, torch.float32), 1e-2)
    assert ispa.get_device_status() == ispa.ISPA_ERR_NOT_SPD
