"""Host-side checks of the C ABI (no GPU): the library loads, exports every symbol the header
declares, validates arguments before touching the device, and the host-only layer selection
(ISPA summary, section 2, "Dynamic Layer Selection") agrees with the oracle."""
import ctypes
import math
import os
import re
import subprocess

import numpy as np
import pytest

import ispa_inputs as inp
from oracle import ispa_oracle as orc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def ispa():
    from kv_cache_compression_tma_b200 import build, ispa as mod
    if not os.path.exists(mod.LIB_PATH):
        build.build()
    mod.lib()
    return mod


def header_functions():
    text = open(os.path.join(ROOT, "include", "ispa.h")).read()
    return re.findall(r"ISPA_API\s+[\w\s\*]+?\b(ispa_\w+)\s*\(", text)


def test_header_symbols_exported(ispa):
    names = header_functions()
    assert len(names) >= 10
    out = subprocess.run(["nm", "-D", "--defined-only", ispa.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\sT\s+(\w+)", out))
    for n in names:
        assert n in exported, n
        assert hasattr(ispa.lib(), n)
    assert set(ispa.SYMBOLS) == set(names)


def test_version_and_status_strings(ispa):
    assert ispa.version() >= 100
    for s in range(8):
        assert ispa.status_string(s)
    assert "unknown" in ispa.status_string(99)


def test_attn_args_layout_matches_header(ispa):
    # offsets of the C struct on x86-64 (int64 after four int32, pointers 8 bytes)
    A = ispa.AttnArgs
    assert A.n_q.offset == 16 and A.n_kv.offset == 24 and A.q.offset == 48 and A.ld_q.offset == 56
    assert A.k.offset == 64 and A.v.offset == 88 and A.ld_k.offset == 112 and A.ld_v.offset == 136
    assert A.softmax_scale.offset == 160 and A.o_loc.offset == 168 and A.d_out.offset == 208
    assert A.kv_bias.offset == 216 and A.ld_bias.offset == 240
    assert ctypes.sizeof(A) == 264


def _attn_args(ispa, **kw):
    a = ispa.AttnArgs()
    a.dtype, a.n_heads, a.head_dim, a.flags = 0, 2, 64, 0
    a.n_q = 8
    for i in range(3):
        a.n_kv[i] = 8
        a.k[i] = a.v[i] = 0x10000
        a.ld_k[i] = a.ld_v[i] = 128
    a.q, a.ld_q = 0x10000, 128
    a.o_loc = a.o_full = a.lse_loc = a.lse_hist = 0x10000
    a.ld_o = 128
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("field,value,expect", [
    ("dtype", 7, 1), ("n_heads", 0, 1), ("head_dim", 48, 2), ("flags", 4, 1), ("n_q", -1, 1),
    ("ld_q", 100, 1), ("ld_o", 64, 1), ("softmax_scale", -1.0, 1), ("softmax_scale", float("nan"), 1),
    ("q", 0x10001, 1), ("o_loc", None, 1), ("lse_loc", None, 1),
])
def test_attention_argument_validation(ispa, field, value, expect):
    a = _attn_args(ispa, **{field: value})
    assert ispa.lib().ispa_dual_stream_attn(ctypes.byref(a), None) == expect


@pytest.mark.parametrize("field,value", [("head_dim", 32), ("ld_q", 132), ("ld_o", 130), ("q", 0x10008)])
def test_bf16_attention_outside_tensor_core_rules_is_refused(ispa, field, value):
    """A bf16 call the tensor-core kernel cannot take returns UNSUPPORTED before touching the device
    (no silent CUDA-core fallback); the CUDA-core kernel is only reached when asked for by flag."""
    a = _attn_args(ispa, **{field: value})
    n0 = ispa.launch_count()
    assert ispa.lib().ispa_dual_stream_attn(ctypes.byref(a), None) == ispa.ISPA_ERR_UNSUPPORTED
    assert ispa.launch_count() == n0
    if not _has_gpu():
        # with the flag the call gets past the refusal and needs a device, which this host lacks
        b = _attn_args(ispa, flags=ispa.ISPA_ATTN_CUDA_CORES, **{field: value})
        assert ispa.lib().ispa_dual_stream_attn(ctypes.byref(b), None) == ispa.ISPA_ERR_CUDA


def _has_gpu():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def test_attention_rejects_empty_local_branch(ispa):
    a = _attn_args(ispa)
    a.n_kv[0] = 0
    a.n_kv[1] = 0
    assert ispa.lib().ispa_dual_stream_attn(ctypes.byref(a), None) == ispa.ISPA_ERR_INVALID_ARG
    a = _attn_args(ispa)
    a.k[2] = None
    assert ispa.lib().ispa_dual_stream_attn(ctypes.byref(a), None) == ispa.ISPA_ERR_INVALID_ARG
    assert ispa.lib().ispa_dual_stream_attn(None, None) == ispa.ISPA_ERR_INVALID_ARG


def test_stats_and_absorb_argument_validation(ispa):
    L = ispa.lib()
    p = 0x10000
    assert L.ispa_accum_stats(5, p, p, 8, 64, 64, 0, p, p, p, None) == 1          # dtype
    assert L.ispa_accum_stats(0, p, p, 8, 64, 32, 0, p, p, p, None) == 1          # lda < d
    assert L.ispa_accum_stats(0, p, p, 8, 64, 64, 8, p, p, p, None) == 1          # flags
    assert L.ispa_accum_stats(0, None, p, 8, 64, 64, 0, p, p, p, None) == 1       # null input
    assert L.ispa_accum_stats(0, p, p, -1, 64, 64, 0, p, p, p, None) == 1         # m < 0
    assert L.ispa_absorb(p, p, p, 0, p, 60, 0.1, 0, p, p, None, p, 1 << 30, None) == 1   # d % 16
    assert L.ispa_absorb(p, p, p, 0, p, 64, -1.0, 0, p, p, None, p, 1 << 30, None) == 1  # lambda < 0
    assert L.ispa_absorb(p, p, p, 0, p, 64, 0.1, 4, p, p, None, p, 1 << 30, None) == 1   # WNEW without w_new
    assert L.ispa_absorb(p, p, p, 0, p, 64, 0.1, 0, p, p, None, p + 16, 1 << 30, None) == 1  # ws alignment
    assert L.ispa_absorb(p, p, p, 0, p, 64, 0.1, 0, p, p, None, p, 16, None) == 1        # ws too small


def test_project_argument_validation(ispa):
    L = ispa.lib()
    p = 0x10000
    assert L.ispa_project(7, p, 8, 64, 64, p, 128, 128, 0, p, 128, None) == 1      # dtype
    assert L.ispa_project(0, p, 8, 64, 64, p, 128, 128, 1, p, 128, None) == 1      # flags
    assert L.ispa_project(0, p, -1, 64, 64, p, 128, 128, 0, p, 128, None) == 1     # m < 0
    assert L.ispa_project(0, p, 8, 64, 32, p, 128, 128, 0, p, 128, None) == 1      # lda < d_in
    assert L.ispa_project(0, p, 8, 64, 64, p, 128, 64, 0, p, 128, None) == 1       # ldw < d_out
    assert L.ispa_project(0, p, 8, 64, 64, p, 128, 32, 2, p, 128, None) == 1       # ldw < d_in (transposed)
    assert L.ispa_project(0, p, 8, 64, 64, p, 128, 128, 0, p, 64, None) == 1       # ldy < d_out
    assert L.ispa_project(0, None, 8, 64, 64, p, 128, 128, 0, p, 128, None) == 1   # null A
    assert L.ispa_project(0, None, 0, 64, 64, None, 128, 128, 0, None, 128, None) == 0  # m == 0: no-op



def test_absorb_static_argument_validation(ispa):
    L = ispa.lib()
    p = 0x10000
    assert L.ispa_absorb_static(p, p, p, 0, p, 2048, 0.1, 0, p, p, None, None) == 2  # wider than its scratch
    assert L.ispa_absorb_static(p, p, p, 0, p, 60, 0.1, 0, p, p, None, None) == 1    # d % 16
    assert L.ispa_absorb_static(p, p, p, 0, p, 8, 0.1, 0, p, p, None, None) == 1     # d < 16


def test_w8a8_argument_validation(ispa):
    """ispa_quantize_e4m3 and ispa_project_w8a8 (reading 16) refuse bad shapes, flags, null and
    misaligned pointers before any device work; empty problems are no-ops."""
    L = ispa.lib()
    p = 0x10000
    q = L.ispa_quantize_e4m3
    assert q(5, p, 8, 64, 64, 0, p, 64, p, None) == 1           # dtype
    assert q(0, p, 8, 64, 64, 2, p, 64, p, None) == 1           # flags
    assert q(0, p, -1, 64, 64, 0, p, 64, p, None) == 1          # rows < 0
    assert q(0, p, 8, 64, 32, 0, p, 64, p, None) == 1           # ldx < cols
    assert q(0, p, 8, 64, 64, 0, p, 32, p, None) == 1           # ldq < cols (per-row codes)
    assert q(0, p, 96, 64, 64, 1, p, 64, p, None) == 1          # ldq < rows (transposed per-column codes)
    assert q(0, None, 8, 64, 64, 0, p, 64, p, None) == 1        # null input
    assert q(0, p + 1, 8, 64, 64, 0, p, 64, p, None) == 1       # bf16 input not 2-byte aligned
    assert q(1, p + 2, 8, 64, 64, 0, p, 64, p, None) == 1       # fp32 input not 4-byte aligned
    assert q(0, p, 8, 64, 64, 0, p, 64, p + 2, None) == 1       # scales not 4-byte aligned
    assert q(0, None, 0, 64, 64, 0, None, 64, None, None) == 0  # rows == 0: no-op
    assert q(0, None, 8, 0, 0, 0, None, 0, None, None) == 0     # cols == 0: no-op
    w = L.ispa_project_w8a8
    assert w(p, p, -1, 64, 64, p, p, 64, 64, p, 64, None) == 1     # m < 0
    assert w(p, p, 8, 0, 64, p, p, 64, 64, p, 64, None) == 1       # d_in < 1
    assert w(p, p, 8, 64, 32, p, p, 64, 64, p, 64, None) == 1      # lda < d_in
    assert w(p, p, 8, 64, 64, p, p, 64, 32, p, 64, None) == 1      # ldw < d_in
    assert w(p, p, 8, 64, 64, p, p, 64, 64, p, 32, None) == 1      # ldy < d_out
    assert w(None, p, 8, 64, 64, p, p, 64, 64, p, 64, None) == 1   # null codes
    assert w(p, p + 1, 8, 64, 64, p, p, 64, 64, p, 64, None) == 1  # row scales misaligned
    assert w(p, p, 8, 64, 64, p, p, 64, 64, p + 1, 64, None) == 1  # bf16 output misaligned
    assert w(None, None, 0, 64, 64, None, None, 64, 64, None, 64, None) == 0  # m == 0: no-op


def test_tempcache_argument_validation(ispa):
    """ispa_tempcache_match / ispa_tempcache_merge (FAST-AR page, section 2 A) refuse unsupported
    head sizes and bad shapes, bounds, pointers and thresholds before any device work."""
    L = ispa.lib()
    p = 0x10000
    m = L.ispa_tempcache_match
    # (n_heads, head_dim, k_new, n_new, ld_new, k_cache, n_cache, ld_cache, inv_norm, ld_state, idx, sim, stream)
    assert m(2, 32, p, 8, 64, p, 16, 64, p, 16, p, p, None) == 2          # head_dim not 64 / 128
    assert m(0, 64, p, 8, 128, p, 16, 128, p, 16, p, p, None) == 2        # no heads
    assert m(2, 64, p, -1, 128, p, 16, 128, p, 16, p, p, None) == 1       # n_new < 0
    assert m(2, 64, p, 8, 128, p, 1 << 20, 128, p, 1 << 20, p, p, None) == 1  # cache bound
    assert m(2, 64, None, 8, 128, p, 16, 128, p, 16, p, p, None) == 1     # null new keys
    assert m(2, 64, p, 8, 64, p, 16, 128, p, 16, p, p, None) == 1         # ld_new < n_heads * head_dim
    assert m(2, 64, p, 8, 132, p, 16, 128, p, 16, p, p, None) == 1        # ld_new not a multiple of 8
    assert m(2, 64, p + 8, 8, 128, p, 16, 128, p, 16, p, p, None) == 1    # new keys not 16-byte aligned
    assert m(2, 64, p, 8, 128, None, 16, 128, p, 16, p, p, None) == 1     # null cache with entries
    assert m(2, 64, p, 8, 128, p, 16, 128, p, 8, p, p, None) == 1         # ld_state < n_cache
    assert m(2, 64, None, 0, 128, None, 16, 128, None, 16, None, None, None) == 0  # no new tokens: no-op
    g = L.ispa_tempcache_merge
    nan = float("nan")
    # (n_heads, head_dim, k_cache, v_cache, ld_cache, capacity, n_cache, count, bias, inv_norm, ld_state,
    #  n_valid, k_new, v_new, n_new, ld_new, idx, sim, threshold, stream)
    ok = (2, 64, p, p, 128, 64, 16, p, p, p, 64, p, p, p, 8, 128, p, p, 0.9, None)
    def call(**kw):
        names = ("n_heads", "head_dim", "k_cache", "v_cache", "ld_cache", "capacity", "n_cache", "count", "bias",
                 "inv_norm", "ld_state", "n_valid", "k_new", "v_new", "n_new", "ld_new", "idx", "sim", "threshold",
                 "stream")
        a = dict(zip(names, ok))
        a.update(kw)
        return g(*(a[n] for n in names))
    assert call(head_dim=48) == 2                 # head_dim not a multiple of 32
    assert call(head_dim=160) == 2                # head_dim > 128
    assert call(capacity=20) == 1                 # capacity < n_cache + n_new
    assert call(n_new=-1) == 1
    assert call(threshold=nan) == 1
    assert call(n_new=5000, capacity=6000, ld_state=6000) == 2  # one frame beyond the merge's sort size
    assert call(bias=None) == 1
    assert call(ld_cache=64) == 1                 # ld_cache < n_heads * head_dim
    assert call(ld_state=32) == 1                 # ld_state < capacity
    assert call(k_new=p + 1) == 1                 # bf16 keys misaligned
    assert call(sim=p + 2) == 1                   # similarities misaligned
    assert call(n_new=0, k_cache=None) == 0       # no new tokens: no-op

def test_kv_accounting():
    from kv_cache_compression_tma_b200 import llayer
    kv = llayer.kv_bytes(1560, 4680, 14040, 12, 128, 2)
    assert kv["kept"] == (1560 + 4680) * 2 * 12 * 128 * 2
    assert kv["history"] == 14040 * 2 * 12 * 128 * 2
    s = llayer.kv_savings([3, 1, 3, 7], 30, kv)   # duplicates count once
    assert s["kv_bytes_freed"] == 3 * kv["history"]
    assert s["kv_bytes_all_full"] == 30 * (kv["kept"] + kv["history"])
    # half the layers as L-Layers free half of the history share of the cache
    h = llayer.kv_savings(range(15), 30, kv)["kv_freed_frac"]
    assert abs(h - 0.5 * 14040 / (1560 + 4680 + 14040)) < 1e-12


def test_workspace_size(ispa):
    for d in (64, 1536, 5120):
        n = ispa.absorb_workspace_size(d)
        assert n >= 4 * 4 * d * d
    with pytest.raises(ispa.IspaError):
        ispa.absorb_workspace_size(20)


def test_select_layers_matches_oracle(ispa):
    for trial in range(50):
        L = 1 + trial % 40
        eps = inp.gaussian((L,), 31, trial) ** 2
        if trial % 7 == 0:
            eps[::3] = eps[0]  # ties
        for k in sorted({0, L // 2, L, min(L, 3)}):
            idx, mask, st = ispa.select_layers(eps, k)
            assert st == 0
            assert list(idx) == list(orc.select_layers(list(eps), k))
            assert mask.sum() == k and all(mask[i] == 1 for i in idx)


def test_select_layers_nan_and_bounds(ispa):
    idx, mask, st = ispa.select_layers([float("nan"), 3.0, 1.0], 2)
    assert list(idx) == [1, 2] and st == 0
    idx, mask, st = ispa.select_layers([float("nan"), 3.0, 1.0], 3)
    assert list(idx) == [0, 1, 2] and st == ispa.ISPA_ERR_NONFINITE
    with pytest.raises(ispa.IspaError):
        ispa.select_layers([1.0, 2.0], 3)
    with pytest.raises(ispa.IspaError):
        ispa.select_layers([1.0, 2.0], -1)


def test_select_layers_thirty_layer_shape(ispa):
    """30 layers, K = 15 (the 1.3B-like warmup's selection)."""
    eps = inp.gaussian((30,), 5, 5) ** 2 + 1.0
    idx, mask, st = ispa.select_layers(eps, 15)
    assert list(idx) == list(orc.select_layers(list(eps), 15))
    assert list(np.flatnonzero(mask)) == list(idx)
