"""The seeded input recipe shared by the oracle and the GPU path (CPU only): bf16 rounding, the AR(1)
K/V timelines, the query scale per layer, row sampling and the workload geometry."""
import numpy as np
import pytest

import ispa_inputs as inp


def test_round_bf16_matches_torch_round_to_nearest_even():
    import torch
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(3.0),
        (rng.standard_normal(2000) * 1e-38).astype(np.float32),            # subnormal range
        np.array([0.0, -0.0, 1.0, -2.5, 3.3895314e38, -3.3895314e38, np.inf, -np.inf], dtype=np.float32),
    ])
    # exact ties: a bf16 value plus half an ulp of bf16 (low 16 bits 0x8000), both parities
    base = rng.standard_normal(2000).astype(np.float32).view(np.uint32) & np.uint32(0xFFFF0000)
    ties = (base | np.uint32(0x8000)).view(np.float32)
    x = np.concatenate([x, ties])
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    got = inp.round_bf16(x)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_ar1_timeline_statistics():
    wl = inp.WORKLOADS["l1_3b"]
    t = inp.kv_timeline(wl, 0, "k", seed=1, n_frames=6).astype(np.float64)
    # stationary N(0, 1) per element, lag-1 correlation rho between frames
    assert abs(t.mean()) < 0.01
    assert abs(t.var() - 1.0) < 0.02
    c = np.mean(t[1:] * t[:-1]) / np.sqrt(np.mean(t[1:] ** 2) * np.mean(t[:-1] ** 2))
    assert c == pytest.approx(wl.rho, abs=0.01)
    # deterministic in the seed, different across layers and between K and V
    assert np.array_equal(t, inp.kv_timeline(wl, 0, "k", seed=1, n_frames=6))
    assert not np.array_equal(t[0], inp.kv_timeline(wl, 1, "k", seed=1, n_frames=1)[0])
    assert not np.array_equal(t[0], inp.kv_timeline(wl, 0, "v", seed=1, n_frames=1)[0])


def test_per_layer_query_scale_spreads_layers():
    wl = inp.WORKLOADS["warm30"]
    s = np.array([inp.logit_scale(wl, l, 0) for l in range(wl.n_layers)])
    assert s.min() == pytest.approx(0.75 * wl.logit_std) and s.max() == pytest.approx(1.25 * wl.logit_std)
    assert len(np.unique(s)) == wl.n_layers          # a permutation: every layer its own scale
    assert inp.logit_scale(inp.WORKLOADS["l1_3b"], 0, 0) == inp.WORKLOADS["l1_3b"].logit_std


def test_sample_rows():
    r = inp.sample_rows(4680, 96, seed=3)
    assert len(r) == 96 and len(np.unique(r)) == 96 and np.all(np.diff(r) > 0)
    assert r[-1] == 4679 and r[0] >= 0
    assert np.array_equal(r, inp.sample_rows(4680, 96, seed=3))
    assert np.array_equal(inp.sample_rows(10, 50), np.arange(10))


def test_workload_geometry():
    wl = inp.WORKLOADS["l1_3b"]
    assert (wl.d, wl.n_heads, wl.head_dim) == (1536, 12, 128)
    assert wl.n_q(0) == 4680 and (wl.n_sink, wl.n_local(0), wl.n_hist(0)) == (1560, 4680, 14040)
    w30 = inp.WORKLOADS["warm30"]
    assert w30.n_layers == 30 and w30.k_select == 15
    assert [w30.n_hist(c) for c in range(len(w30.chunks))] == [0, 4680, 9360, 14040]
    l14 = inp.WORKLOADS["l14b"]
    assert (l14.d, l14.n_layers, l14.k_select) == (5120, 40, 20)
    lh = inp.get_workload("longhist60")
    assert lh.n_hist(0) == 60 * 1560 and lh.rho == 0.95
    x = inp.attention_inputs(wl, 0, 0, seed=0)
    assert x["q"].shape == (4680, 12, 128) and x["k_hist"].shape == (14040, 12, 128)
    assert np.array_equal(x["q"], inp.round_bf16(x["q"]))  # bf16 workloads hold bf16 values
