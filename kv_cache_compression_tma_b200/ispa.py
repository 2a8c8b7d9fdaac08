"""ctypes binding of libispa.so (the C ABI in include/ispa.h).

Argument marshalling only: every step of the hot path runs in the library's CUDA kernels.  PyTorch
provides device memory and the current stream.  If the library is missing the calls raise; there
is no fallback.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libispa.so")

ISPA_OK, ISPA_ERR_INVALID_ARG, ISPA_ERR_UNSUPPORTED, ISPA_ERR_CUDA = 0, 1, 2, 3
ISPA_ERR_NOT_SPD, ISPA_ERR_NONFINITE, ISPA_ERR_TIMEOUT, ISPA_ERR_INTERNAL = 4, 5, 6, 7
ISPA_BF16, ISPA_F32 = 0, 1
ISPA_ATTN_CUDA_CORES = 0x1
ISPA_STATS_ZERO, ISPA_STATS_SECOND_IS_FULL = 0x1, 0x2
ISPA_LAMBDA_REL, ISPA_W_TRANSPOSED, ISPA_WRITE_WNEW = 0x1, 0x2, 0x4
ISPA_TEST_ATTN_NO_LOADS = 0x1
ISPA_QUANT_COLUMNS = 0x1

SYMBOLS = ("ispa_dual_stream_attn", "ispa_accum_stats", "ispa_absorb_workspace_size", "ispa_absorb",
           "ispa_absorb_static", "ispa_project", "ispa_quantize_e4m3", "ispa_project_w8a8", "ispa_tempcache_match",
           "ispa_tempcache_merge", "ispa_select_layers",
           "ispa_get_device_status",
           "ispa_peek_device_status_bits", "ispa_test_set_flags",
           "ispa_status_string", "ispa_version", "ispa_launch_count")


class IspaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


class AttnArgs(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int32), ("n_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("flags", ctypes.c_int32), ("n_q", ctypes.c_int64), ("n_kv", ctypes.c_int64 * 3),
        ("q", ctypes.c_void_p), ("ld_q", ctypes.c_int64),
        ("k", ctypes.c_void_p * 3), ("v", ctypes.c_void_p * 3),
        ("ld_k", ctypes.c_int64 * 3), ("ld_v", ctypes.c_int64 * 3),
        ("softmax_scale", ctypes.c_float), ("reserved0", ctypes.c_float),
        ("o_loc", ctypes.c_void_p), ("o_full", ctypes.c_void_p), ("ld_o", ctypes.c_int64),
        ("lse_loc", ctypes.c_void_p), ("lse_hist", ctypes.c_void_p), ("d_out", ctypes.c_void_p),
        ("kv_bias", ctypes.c_void_p * 3), ("ld_bias", ctypes.c_int64 * 3),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libispa.so (built in-tree by kv_cache_compression_tma_b200.build); raise if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m kv_cache_compression_tma_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.ispa_dual_stream_attn.argtypes = [ctypes.POINTER(AttnArgs), ctypes.c_void_p]
        L.ispa_accum_stats.argtypes = [ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                       ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_void_p,
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        L.ispa_absorb_workspace_size.argtypes = [ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]
        L.ispa_absorb.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                                  ctypes.c_int32, ctypes.c_float, ctypes.c_uint32, ctypes.c_void_p, ctypes.c_void_p,
                                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
        L.ispa_absorb_static.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                         ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_uint32,
                                         ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        L.ispa_project.argtypes = [ctypes.c_int32, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int64,
                                   ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_void_p,
                                   ctypes.c_int64, ctypes.c_void_p]
        L.ispa_quantize_e4m3.argtypes = [ctypes.c_int32, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                                         ctypes.c_int64, ctypes.c_uint32, ctypes.c_void_p, ctypes.c_int64,
                                         ctypes.c_void_p, ctypes.c_void_p]
        L.ispa_project_w8a8.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                                        ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                        ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
        L.ispa_tempcache_match.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_int64,
                                           ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                           ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.c_void_p]
        L.ispa_tempcache_merge.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p]
        L.ispa_select_layers.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.c_int32, ctypes.c_int32,
                                         ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_uint8)]
        L.ispa_get_device_status.argtypes = [ctypes.c_void_p]
        L.ispa_peek_device_status_bits.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
        L.ispa_test_set_flags.argtypes = [ctypes.c_uint32]
        L.ispa_status_string.argtypes = [ctypes.c_int32]
        L.ispa_status_string.restype = ctypes.c_char_p
        L.ispa_version.restype = ctypes.c_int32
        L.ispa_launch_count.restype = ctypes.c_uint64
        for name in ("ispa_dual_stream_attn", "ispa_accum_stats", "ispa_absorb_workspace_size", "ispa_absorb",
                     "ispa_absorb_static", "ispa_select_layers", "ispa_get_device_status", "ispa_peek_device_status_bits",
                     "ispa_test_set_flags", "ispa_quantize_e4m3", "ispa_project_w8a8", "ispa_tempcache_match",
                     "ispa_tempcache_merge"):
            getattr(L, name).restype = ctypes.c_int32
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().ispa_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != ISPA_OK:
        raise IspaError(status, what)


def _stream(stream=None) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return ISPA_BF16
    if t.dtype == torch.float32:
        return ISPA_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _on_current_device(*tensors):
    """The library resolves its per-device state (status word, scratch, streams) from the CURRENT
    device, so every tensor of a call must live there."""
    import torch
    cur = torch.cuda.current_device()
    for t in tensors:
        if t is not None and (t.device.type != "cuda" or t.device.index != cur):
            raise ValueError(f"tensor on {t.device}, but the current CUDA device is cuda:{cur}; "
                             f"call under `with torch.cuda.device(...)`")


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _row_stride(t, what: str) -> int:
    """Token/row stride of a [tokens, H, hd] or [rows, d] tensor whose inner dims are dense."""
    if t.dim() == 3:
        if t.stride(2) != 1 or t.stride(1) != t.shape[2]:
            raise ValueError(f"{what}: heads and head_dim must be contiguous")
    elif t.dim() == 2:
        if t.stride(1) != 1:
            raise ValueError(f"{what}: columns must be contiguous")
    else:
        raise ValueError(f"{what}: expected 2 or 3 dims")
    if t.shape[0] <= 1:  # a single row: its stride is irrelevant, report the dense row length
        return int(np.prod(t.shape[1:]))
    return int(t.stride(0))


def dual_stream_attn(q, k_sink, v_sink, k_loc, v_loc, k_hist, v_hist, *, o_loc=None, o_full=None, lse_loc=None,
                     lse_hist=None, d_out=None, want_delta: bool = True, softmax_scale: float = 0.0,
                     cuda_cores: bool = False, kv_bias=(None, None, None), stream=None) -> dict:
    """ispa_dual_stream_attn on torch CUDA tensors.

    q, k_*, v_*: [tokens, H, hd] (bf16 or fp32).  Outputs (allocated if not given): o_loc, o_full and
    (if want_delta) d = O_full - O_loc as [n_q, H*hd] in q's dtype; lse_loc, lse_hist fp32 [H, n_q].
    kv_bias: optional per-segment fp32 [H, n_kv] additive logit biases (natural log), e.g. the log group
    sizes of a TempCache-merged history.
    """
    import torch
    _on_current_device(q, k_sink, v_sink, k_loc, v_loc, k_hist, v_hist, o_loc, o_full, lse_loc, lse_hist, d_out,
                       *kv_bias)
    n_q, H, hd = q.shape
    d = H * hd
    dev = q.device
    if o_loc is None:
        o_loc = torch.empty((n_q, d), dtype=q.dtype, device=dev)
    if o_full is None:
        o_full = torch.empty((n_q, d), dtype=q.dtype, device=dev)
    if d_out is None and want_delta:
        d_out = torch.empty((n_q, d), dtype=q.dtype, device=dev)
    if lse_loc is None:
        lse_loc = torch.empty((H, n_q), dtype=torch.float32, device=dev)
    if lse_hist is None:
        lse_hist = torch.empty((H, n_q), dtype=torch.float32, device=dev)
    a = AttnArgs()
    a.dtype = _dtype_code(q)
    a.n_heads, a.head_dim = H, hd
    a.flags = ISPA_ATTN_CUDA_CORES if cuda_cores else 0
    a.n_q = n_q
    a.q, a.ld_q = _ptr(q), _row_stride(q, "q") if n_q else d
    for i, (k, v) in enumerate(((k_sink, v_sink), (k_loc, v_loc), (k_hist, v_hist))):
        a.n_kv[i] = k.shape[0]
        if k.shape[0]:
            a.k[i], a.v[i] = _ptr(k), _ptr(v)
            a.ld_k[i], a.ld_v[i] = _row_stride(k, "k"), _row_stride(v, "v")
        else:
            a.k[i] = a.v[i] = None
            a.ld_k[i] = a.ld_v[i] = d
    a.softmax_scale = float(softmax_scale)
    a.o_loc, a.o_full, a.d_out = _ptr(o_loc), _ptr(o_full), _ptr(d_out)
    a.ld_o = _row_stride(o_loc, "o_loc") if n_q else d
    a.lse_loc, a.lse_hist = _ptr(lse_loc), _ptr(lse_hist)
    for i, bt in enumerate(kv_bias):
        if bt is not None:
            if bt.dtype != torch.float32 or bt.dim() != 2 or bt.stride(1) != 1:
                raise ValueError("kv_bias entries must be fp32 [H, n_kv] with contiguous columns")
            a.kv_bias[i], a.ld_bias[i] = _ptr(bt), int(bt.stride(0))
    _check(lib().ispa_dual_stream_attn(ctypes.byref(a), _stream(stream)), "ispa_dual_stream_attn")
    return {"o_loc": o_loc, "o_full": o_full, "d": d_out, "lse_loc": lse_loc, "lse_hist": lse_hist}


def accum_stats(a_loc, a_second, G, R, S, *, second_is_full: bool = False, zero: bool = False, stream=None):
    """ispa_accum_stats: G/R/S (fp32 [d, d]) (+)= A_loc^T A_loc, A_loc^T D, D^T D over the rows given."""
    _on_current_device(a_loc, a_second, G, R, S)
    m, d = a_loc.shape
    flags = (ISPA_STATS_ZERO if zero else 0) | (ISPA_STATS_SECOND_IS_FULL if second_is_full else 0)
    lda = _row_stride(a_loc, "a_loc") if m else d
    if m and _row_stride(a_second, "a_second") != lda:
        raise ValueError("a_loc and a_second must share a row stride")
    _check(lib().ispa_accum_stats(_dtype_code(a_loc), _ptr(a_loc), _ptr(a_second), m, d, lda, flags, _ptr(G),
                                  _ptr(R), _ptr(S), _stream(stream)), "ispa_accum_stats")
    return G, R, S


def absorb_workspace_size(d: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().ispa_absorb_workspace_size(int(d), ctypes.byref(n)), "ispa_absorb_workspace_size")
    return int(n.value)


def absorb(G, R, S, W, lam: float, *, lam_rel: bool = False, w_transposed: bool = False, dW=None, eps=None,
           w_new=None, write_wnew: bool = False, ws=None, stream=None) -> dict:
    """ispa_absorb: dW = (G + lam I)^-1 R W and eps = {eps, eps_rel, lam, <W, S W>} (fp64, on device)."""
    import torch
    _on_current_device(G, R, S, W, dW, eps, w_new, ws)
    d = G.shape[0]
    dev = G.device
    if dW is None:
        dW = torch.empty((d, d), dtype=torch.float32, device=dev)
    if eps is None:
        eps = torch.empty((4,), dtype=torch.float64, device=dev)
    if ws is None:
        ws = torch.empty((absorb_workspace_size(d),), dtype=torch.uint8, device=dev)
    if write_wnew and w_new is None:
        w_new = torch.empty_like(W)
    flags = (ISPA_LAMBDA_REL if lam_rel else 0) | (ISPA_W_TRANSPOSED if w_transposed else 0) | \
            (ISPA_WRITE_WNEW if write_wnew else 0)
    _check(lib().ispa_absorb(_ptr(G), _ptr(R), _ptr(S), _dtype_code(W), _ptr(W), d, float(lam), flags, _ptr(dW),
                             _ptr(eps), _ptr(w_new), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "ispa_absorb")
    return {"dW": dW, "eps": eps, "w_new": w_new, "ws": ws}


ABSORB_STATIC_MAX_D = 1536


def absorb_static(G, R, S, W, lam: float, *, lam_rel: bool = False, w_transposed: bool = False, dW=None,
                  eps=None, w_new=None, write_wnew: bool = False, stream=None) -> dict:
    """ispa_absorb_static: the absorb without a caller workspace (library-held scratch, d <= 1536).
    For callers that cannot allocate device memory at absorb time; the outputs are still the caller's."""
    import torch
    _on_current_device(G, R, S, W, dW, eps, w_new)
    d = G.shape[0]
    dev = G.device
    if dW is None:
        dW = torch.empty((d, d), dtype=torch.float32, device=dev)
    if eps is None:
        eps = torch.empty((4,), dtype=torch.float64, device=dev)
    if write_wnew and w_new is None:
        w_new = torch.empty_like(W)
    flags = (ISPA_LAMBDA_REL if lam_rel else 0) | (ISPA_W_TRANSPOSED if w_transposed else 0) | \
            (ISPA_WRITE_WNEW if write_wnew else 0)
    _check(lib().ispa_absorb_static(_ptr(G), _ptr(R), _ptr(S), _dtype_code(W), _ptr(W), d, float(lam), flags,
                                    _ptr(dW), _ptr(eps), _ptr(w_new), _stream(stream)), "ispa_absorb_static")
    return {"dW": dW, "eps": eps, "w_new": w_new}


def project(A, W, *, w_transposed: bool = False, out=None, stream=None):
    """ispa_project: Y = A W (or A W^T for a torch-Linear-layout W) with A [m, d_in] and W [d_in, d_out]
    ([d_out, d_in] when w_transposed); bf16 runs the tensor-core kernel, fp32 the CUDA-core one."""
    import torch
    _on_current_device(A, W, out)
    if A.dtype != W.dtype:
        raise ValueError("A and W must have the same dtype")
    m, d_in = A.shape
    d_out = W.shape[0] if w_transposed else W.shape[1]
    if (W.shape[1] if w_transposed else W.shape[0]) != d_in:
        raise ValueError("W does not match A's width")
    if out is None:
        out = torch.empty((m, d_out), dtype=A.dtype, device=A.device)
    flags = ISPA_W_TRANSPOSED if w_transposed else 0
    _check(lib().ispa_project(_dtype_code(A), _ptr(A), m, d_in, _row_stride(A, "A"), _ptr(W), d_out,
                              _row_stride(W, "W"), flags, _ptr(out), _row_stride(out, "out"), _stream(stream)),
           "ispa_project")
    return out


def quantize_e4m3(X, *, columns: bool = False, q=None, scale=None, stream=None):
    """ispa_quantize_e4m3: fp8 E4M3 codes (torch.uint8) and fp32 scales of X [rows, cols] (bf16 or
    fp32).  Per row by default: q [rows, cols], scale [rows].  columns=True: per column, q written
    transposed [cols, rows] (the K-major weight layout of project_w8a8), scale [cols]."""
    import torch
    _on_current_device(X, q, scale)
    rows, cols = X.shape
    if q is None:
        q = torch.empty((cols, rows) if columns else (rows, cols), dtype=torch.uint8, device=X.device)
    if scale is None:
        scale = torch.empty((cols if columns else rows,), dtype=torch.float32, device=X.device)
    ldx = _row_stride(X, "X") if rows else cols
    ldq = _row_stride(q, "q") if q.shape[0] > 1 else q.shape[1]
    _check(lib().ispa_quantize_e4m3(_dtype_code(X), _ptr(X), rows, cols, ldx, ISPA_QUANT_COLUMNS if columns else 0,
                                    _ptr(q), ldq, _ptr(scale), _stream(stream)), "ispa_quantize_e4m3")
    return q, scale


def project_w8a8(qa, sa, qw, sw, *, out=None, stream=None):
    """ispa_project_w8a8: Y = diag(sa) (qa qw^T) diag(sw) in bf16, with qa [m, d_in] and qw [d_out, d_in]
    E4M3 codes (torch.uint8) from quantize_e4m3."""
    import torch
    _on_current_device(qa, sa, qw, sw, out)
    m, d_in = qa.shape
    d_out = qw.shape[0]
    if qw.shape[1] != d_in:
        raise ValueError("qw does not match qa's width")
    if out is None:
        out = torch.empty((m, d_out), dtype=torch.bfloat16, device=qa.device)
    _check(lib().ispa_project_w8a8(_ptr(qa), _ptr(sa), m, d_in, _row_stride(qa, "qa"), _ptr(qw), _ptr(sw), d_out,
                                   _row_stride(qw, "qw"), _ptr(out), _row_stride(out, "out"), _stream(stream)),
           "ispa_project_w8a8")
    return out


class TempCache:
    """A TempCache-merged KV segment on the device (FAST-AR TempCache): per-head entries with
    representative keys, mean values, group sizes, their logs as the attention bias, and inverse key
    norms; see ispa_tempcache_match / ispa_tempcache_merge in include/ispa.h."""

    def __init__(self, n_heads: int, head_dim: int, capacity: int, device="cuda"):
        import torch
        self.n_heads, self.head_dim, self.capacity = n_heads, head_dim, capacity
        ld_state = (capacity + 3) // 4 * 4
        self.k = torch.zeros((capacity, n_heads, head_dim), dtype=torch.bfloat16, device=device)
        self.v = torch.zeros_like(self.k)
        self.count = torch.zeros((n_heads, ld_state), dtype=torch.int32, device=device)
        self.bias = torch.full((n_heads, ld_state), float("-inf"), dtype=torch.float32, device=device)
        self.inv_norm = torch.full((n_heads, ld_state), -1.0, dtype=torch.float32, device=device)
        self.n_valid = torch.zeros((n_heads,), dtype=torch.int32, device=device)
        self.n_cache = 0  # bound on every head's entry count: the segment length to attend over

    def match(self, k_new, idx=None, sim=None, stream=None):
        import torch
        _on_current_device(k_new, self.k, idx, sim)
        n_new = k_new.shape[0]
        if idx is None:
            idx = torch.empty((self.n_heads, n_new), dtype=torch.int32, device=k_new.device)
        if sim is None:
            sim = torch.empty((self.n_heads, n_new), dtype=torch.float32, device=k_new.device)
        ld_new = _row_stride(k_new, "k_new") if n_new else self.n_heads * self.head_dim
        _check(lib().ispa_tempcache_match(self.n_heads, self.head_dim, _ptr(k_new), n_new, ld_new, _ptr(self.k),
                                          self.n_cache, self.n_heads * self.head_dim, _ptr(self.inv_norm),
                                          self.count.stride(0), _ptr(idx), _ptr(sim), _stream(stream)),
               "ispa_tempcache_match")
        return idx, sim

    def merge(self, k_new, v_new, idx, sim, threshold: float, stream=None):
        _on_current_device(k_new, v_new, idx, sim, self.k)
        n_new = k_new.shape[0]
        ld_new = _row_stride(k_new, "k_new") if n_new else self.n_heads * self.head_dim
        if n_new and _row_stride(v_new, "v_new") != ld_new:
            raise ValueError("k_new and v_new must share a row stride")
        _check(lib().ispa_tempcache_merge(self.n_heads, self.head_dim, _ptr(self.k), _ptr(self.v),
                                          self.n_heads * self.head_dim, self.capacity, self.n_cache, _ptr(self.count),
                                          _ptr(self.bias), _ptr(self.inv_norm), self.count.stride(0),
                                          _ptr(self.n_valid), _ptr(k_new), _ptr(v_new), n_new, ld_new, _ptr(idx),
                                          _ptr(sim), float(threshold), _stream(stream)), "ispa_tempcache_merge")
        self.n_cache += n_new

    def add_frame(self, k_new, v_new, threshold: float, stream=None):
        """Match then merge one frame; returns (idx, sim) of the match."""
        idx, sim = self.match(k_new, stream=stream)
        self.merge(k_new, v_new, idx, sim, threshold, stream=stream)
        return idx, sim

    def segment(self):
        """(k, v, bias) views of the live bound, for dual_stream_attn's history segment."""
        n = self.n_cache
        return self.k[:n], self.v[:n], self.bias[:, :n]


def select_layers(eps: Sequence[float], k: int):
    """ispa_select_layers (host): indices of the k lowest-eps layers (ascending index) and a 0/1 mask.
    Returns (idx int32 array, mask uint8 array, status)."""
    e = np.ascontiguousarray(np.asarray(eps, dtype=np.float64))
    n = int(e.shape[0])
    idx = np.zeros((max(k, 1),), dtype=np.int32)
    mask = np.zeros((max(n, 1),), dtype=np.uint8)
    st = lib().ispa_select_layers(e.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), n, int(k),
                                  idx.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                  mask.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)))
    if st not in (ISPA_OK, ISPA_ERR_NONFINITE):
        raise IspaError(st, "ispa_select_layers")
    return idx[:k].copy(), mask[:n].copy(), st


def get_device_status(stream=None) -> int:
    return int(lib().ispa_get_device_status(_stream(stream)))


def test_set_flags(flags: int) -> None:
    """ispa_test_set_flags: process-wide test hooks (0 = off), for tests of the device-status path."""
    _check(lib().ispa_test_set_flags(int(flags)), "ispa_test_set_flags")


def launch_count() -> int:
    return int(lib().ispa_launch_count())


def version() -> int:
    return int(lib().ispa_version())
