"""Inference after T_warm (ISPA section 2, stage 3): the K layers chosen by the dynamic layer
selection become L-Layers, which attend over their local context only (sink tokens + current chunk;
their history K/V are no longer kept) and project with W_new = W + dW; the other layers stay
F-Layers with full attention and W.

Orchestration only: every step runs in libispa's kernels (ispa_dual_stream_attn with an empty history
segment for L-Layers, ispa_project for the projection).  The KV accounting says how many bytes of
history the L-Layers no longer hold, the memory the method frees.
"""
from __future__ import annotations

from typing import Dict, Optional, Sequence

from . import ispa


class LayerWork:
    """Reusable device buffers of one layer forward ([n_q, d] attention outputs, lse rows)."""

    def __init__(self, n_q: int, n_heads: int, head_dim: int, dtype, device="cuda"):
        import torch
        d = n_heads * head_dim
        self.o_loc = torch.empty((n_q, d), dtype=dtype, device=device)
        self.o_full = torch.empty_like(self.o_loc)
        self.lse_loc = torch.empty((n_heads, n_q), dtype=torch.float32, device=device)
        self.lse_hist = torch.empty_like(self.lse_loc)

    def view(self, n: int) -> Dict[str, object]:
        return {"o_loc": self.o_loc[:n], "o_full": self.o_full[:n], "lse_loc": self.lse_loc[:, :n],
                "lse_hist": self.lse_hist[:, :n]}


def layer_forward(q, k_sink, v_sink, k_loc, v_loc, k_hist, v_hist, W, *, llayer: bool, w_transposed: bool = False,
                  work: Optional[LayerWork] = None, out=None, stream=None):
    """One layer's attention and output projection after T_warm.

    F-Layer (llayer False): attention over sink + local + history, y = A_full W.
    L-Layer (llayer True): attention over sink + local only (k_hist / v_hist are ignored and may be
    None), y = A_loc W, where the caller passes W_new as W.
    q and the k/v segments are [tokens, H, hd]; W is [d, d_out] (or [d_out, d] with w_transposed).
    Returns y [n_q, d_out] in the dtype of q.
    """
    n, H, hd = q.shape
    if work is None:
        work = LayerWork(n, H, hd, q.dtype, q.device)
    buf = work.view(n)
    if llayer:
        k_hist = k_loc[:0]
        v_hist = v_loc[:0]
    ispa.dual_stream_attn(q, k_sink, v_sink, k_loc, v_loc, k_hist, v_hist, want_delta=False, stream=stream, **buf)
    a = buf["o_loc"] if llayer else buf["o_full"]
    return ispa.project(a, W, w_transposed=w_transposed, out=out, stream=stream)


def kv_bytes(n_sink: int, n_local: int, n_hist: int, n_heads: int, head_dim: int, elem_bytes: int) -> Dict[str, int]:
    """K and V bytes of one layer's cache at one chunk: the part every layer keeps (sink + local) and
    the history that only an F-Layer keeps."""
    row = 2 * n_heads * head_dim * elem_bytes  # one token's K and V
    return {"kept": (n_sink + n_local) * row, "history": n_hist * row}


def kv_savings(selected: Sequence[int], n_layers: int, per_layer: Dict[str, int]) -> Dict[str, float]:
    """Cache bytes of the whole stack with every layer an F-Layer, the bytes the selected L-Layers
    free, and the freed fraction."""
    total = n_layers * (per_layer["kept"] + per_layer["history"])
    freed = len(set(int(i) for i in selected)) * per_layer["history"]
    return {"kv_bytes_all_full": float(total), "kv_bytes_freed": float(freed),
            "kv_freed_frac": float(freed / total) if total else 0.0}
