"""GPU parity of decomposable dual-stream attention (ISPA summary, section 2, stage 1) against the
fp64 oracle's separate local / full / history passes, through the C ABI.

Tolerances (bf16 inputs, fp32 accumulation, P rounded to bf16 for PV, outputs rounded to bf16):
relative Frobenius error <= 1e-2 for O_loc, O_full and D; max |lse error| <= 2e-3."""
import numpy as np
import pytest

import ispa_inputs as inp
from oracle import ispa_oracle as orc
from gpu_helpers import ATTN_TOL, assert_attention_ok, attention_errors, host, rel, run_attention, torch_dtype

pytestmark = pytest.mark.gpu

L13 = inp.WORKLOADS["l1_3b"]


def small(hd=128, frame=100, sink=40, heads=2, hist=9, chunk_frames=3):
    """The 1.3B-like geometry at reduced size: several 128-key tiles with ragged tails per segment."""
    return inp.Workload(f"small{hd}", heads, hd, frame, sink, chunk_frames, inp._single_chunk(hist, chunk_frames),
                        1, None, 1e-2, 0.9, 2.0, "bf16")


def oracle_for(x, rows=None, with_hist=True):
    """Oracle passes C1 (local), C2 (full) and, unless skipped for time, C3 (history only)."""
    ref = orc.dual_stream(x["q"], x["k_sink"], x["v_sink"], x["k_loc"], x["v_loc"], x["k_hist"], x["v_hist"],
                          rows=rows, with_hist=with_hist)
    ref["with_hist"] = with_hist
    return ref


@pytest.mark.parametrize("hd", [128, 64])
def test_tensor_core_ragged_tiles(cuda_ok, hd):
    wl = small(hd=hd)
    x = inp.attention_inputs(wl, 0, 0, seed=1)
    assert x["q"].shape[0] == 300 and x["k_sink"].shape[0] == 40 and x["k_hist"].shape[0] == 900
    out = run_attention(x, torch_dtype(wl))
    assert_attention_ok(attention_errors(out, oracle_for(x)))


def test_tensor_core_matches_cuda_core_kernel(cuda_ok):
    wl = small()
    x = inp.attention_inputs(wl, 0, 0, seed=2)
    a = run_attention(x, torch_dtype(wl))
    b = run_attention(x, torch_dtype(wl), cuda_cores=True)
    for k in ("o_loc", "o_full", "d"):
        assert rel(host(a[k]), host(b[k])) <= 1e-2, k
    assert np.max(np.abs(host(a["lse_loc"]) - host(b["lse_loc"]))) <= 2e-3


def test_empty_history_is_exact(cuda_ok):
    """No history: lse_hist = -inf, O_full bitwise equal to O_loc, D exactly zero (stage 1: A_full is
    attention over the whole history, which here is empty)."""
    wl = small(hist=0)
    x = inp.attention_inputs(wl, 0, 0, seed=3)
    assert x["k_hist"].shape[0] == 0
    for cuda_cores in (False, True):
        out = run_attention(x, torch_dtype(wl), cuda_cores=cuda_cores)
        assert np.array_equal(host(out["o_full"]), host(out["o_loc"]))
        assert not host(out["d"]).any()
        assert np.all(np.isneginf(host(out["lse_hist"])))
        assert_attention_ok(attention_errors(out, oracle_for(x)))


def test_no_sink_and_single_local_key(cuda_ok):
    wl = small(sink=0)
    x = inp.attention_inputs(wl, 0, 0, seed=4)
    assert x["k_sink"].shape[0] == 0
    assert_attention_ok(attention_errors(run_attention(x, torch_dtype(wl)), oracle_for(x)))
    # one local key, no sink: O_loc equals that key's value row (softmax closed form)
    y = dict(x)
    y["k_loc"], y["v_loc"] = x["k_loc"][:1], x["v_loc"][:1]
    y["q"] = x["q"][:5]
    out = run_attention(y, torch_dtype(wl))
    o_loc = host(out["o_loc"]).reshape(5, wl.n_heads, wl.head_dim)
    assert np.allclose(o_loc, np.repeat(y["v_loc"][:1].astype(np.float64), 5, axis=0), rtol=4e-3, atol=0)
    assert_attention_ok(attention_errors(out, oracle_for(y)))


def test_query_count_below_one_tile(cuda_ok):
    wl = small(frame=20, sink=20, chunk_frames=1, hist=2)
    x = inp.attention_inputs(wl, 0, 0, seed=5)
    assert x["q"].shape[0] == 20
    assert_attention_ok(attention_errors(run_attention(x, torch_dtype(wl)), oracle_for(x)))


def test_tiny_fp32_all_rows(cuda_ok):
    wl = inp.WORKLOADS["tiny"]
    for c in range(2):
        x = inp.attention_inputs(wl, 0, c, seed=0)
        out = run_attention(x, torch_dtype(wl))
        err = attention_errors(out, oracle_for(x))
        # fp32 arithmetic end to end: far inside the bf16 tolerances
        assert err["o_loc"] <= 1e-5 and err["o_full"] <= 1e-5 and err["d"] <= 1e-4, err
        assert err["lse_loc"] <= 1e-4 and err["lse_hist"] <= 1e-4, err


def test_l1_3b_layer_all_rows(cuda_ok):
    """One 1.3B-like layer (4680 queries, 1560 sink + 4680 local + 14040 history keys), every row of
    every head against the oracle."""
    x = inp.attention_inputs(L13, 0, 0, seed=0)
    out = run_attention(x, torch_dtype(L13))
    err = attention_errors(out, oracle_for(x, with_hist=False))
    assert_attention_ok(err)


@pytest.mark.parametrize("frames", [3, 120])
def test_long_history_sampled_rows(cuda_ok, frames):
    """Long-history stress (rho = 0.95, up to 187200 history keys): a seeded sample of rows, which the
    oracle computes one by one (rows are independent)."""
    wl = inp.longhist(frames)
    x = inp.attention_inputs(wl, 0, 0, seed=0)
    out = run_attention(x, torch_dtype(wl))
    rows = inp.sample_rows(wl.n_q(), 96, seed=0, salt=frames)
    ref = oracle_for(x, rows=rows)
    assert_attention_ok(attention_errors(out, ref, rows=rows))


def test_warmup_chunks_sampled_rows(cuda_ok):
    """The 1.3B-like warmup timeline: chunks with 0, 3, 6 and 9 history frames, one layer."""
    wl = inp.WORKLOADS["warm30"]
    tl = (inp.kv_timeline(wl, 3, "k"), inp.kv_timeline(wl, 3, "v"))
    for c in range(4):
        x = inp.attention_inputs(wl, 3, c, seed=0, timelines=tl)
        out = run_attention(x, torch_dtype(wl))
        rows = inp.sample_rows(wl.n_q(c), 64, seed=0, salt=c)
        assert_attention_ok(attention_errors(out, oracle_for(x, rows=rows), rows=rows))
        if c == 0:
            assert np.array_equal(host(out["o_full"]), host(out["o_loc"]))


def test_launch_counter_and_status(cuda_ok):
    from kv_cache_compression_tma_b200 import ispa
    wl = small()
    x = inp.attention_inputs(wl, 0, 0, seed=6)
    n0 = ispa.launch_count()
    run_attention(x, torch_dtype(wl))
    assert ispa.launch_count() == n0 + 1
    assert ispa.get_device_status() == ispa.ISPA_OK
