"""Seeded synthetic inputs for the ISPA hot path.

This module is the one piece shared by the CUDA path's tests/benchmark and by the CPU oracle.
It holds none of the method's arithmetic: it only draws random numbers with the token geometry
of the workloads and rounds them to their storage dtype.

Geometry (ISPA summary, section 2 "Framework Core", stage 1): a streaming video generator emits
chunks of latent frames; every attention call sees three key/value segments

    sink  : the first latent frame's tokens (the "sink" tokens),
    local : the current chunk's tokens (the queries' own frames),
    hist  : every cached frame between the sink and the current chunk.

Recipe (one timeline per layer and per K/V tensor):
  * frame f0 is the sink frame; frames are 1560 tokens (52x30 latent patches) for the 1.3B-
    and 14B-like shapes, 32 tokens for the tiny case (whose sink is tokens 0..15 of f0);
  * K and V follow an AR(1) chain across frames per (token position, head, element):
    x_f = rho * x_{f-1} + sqrt(1 - rho^2) * xi_f, xi ~ N(0,1), x_0 ~ N(0,1);
  * Q is i.i.d. N(0,1) * s, so that the logits q.k / sqrt(head_dim) have std ~= s;
    for the multi-layer warmup shapes layer l uses s_l = 2 * (0.75 + 0.5 * pi(l) / (L-1)) with a
    seeded permutation pi, so that layers differ in how much they lean on the history;
  * W ~ N(0, 1/d) per layer;
  * bf16 workloads round every tensor to bf16 (round-to-nearest-even from float32); the arrays
    returned here are float32 holding exactly those bf16 values, so both sides read identical data.

Seeds: numpy PCG64 seeded by SeedSequence([seed, layer, chunk, tensor-id]) so that any (layer,
chunk) can be regenerated alone.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence

import numpy as np

_T_K, _T_V, _T_Q, _T_W, _T_PERM, _T_ROWS = 1, 2, 3, 4, 5, 6


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    n_heads: int
    head_dim: int
    frame_tokens: int
    n_sink: int
    chunk_frames: int
    # per chunk: the cached history frame indices and the current frame indices (f0 = sink frame)
    chunks: tuple
    n_layers: int
    k_select: Optional[int]
    lam_rel: Optional[float]
    rho: float
    logit_std: float
    dtype: str  # "bf16" or "f32"
    per_layer_scale: bool = False
    description: str = ""

    @property
    def d(self) -> int:
        return self.n_heads * self.head_dim

    def n_q(self, chunk: int = 0) -> int:
        return len(self.chunks[chunk][1]) * self.frame_tokens

    def n_hist(self, chunk: int = 0) -> int:
        return len(self.chunks[chunk][0]) * self.frame_tokens

    def n_local(self, chunk: int = 0) -> int:
        return self.n_q(chunk)

    @property
    def rows_per_layer(self) -> int:
        return sum(self.n_q(c) for c in range(len(self.chunks)))

    @property
    def n_frames(self) -> int:
        return 1 + max(max(list(h) + list(c)) for h, c in self.chunks)


def _warmup_chunks(n_chunks: int, chunk_frames: int):
    out = []
    for c in range(n_chunks):
        cur = tuple(range(1 + chunk_frames * c, 1 + chunk_frames * (c + 1)))
        hist = tuple(range(1, 1 + chunk_frames * c))
        out.append((hist, cur))
    return tuple(out)


def _single_chunk(hist_frames: int, chunk_frames: int):
    return ((tuple(range(1, 1 + hist_frames)), tuple(range(1 + hist_frames, 1 + hist_frames + chunk_frames))),)


def _rolling_tiny():
    # two 1-frame chunks, each with a rolling 3-frame history window
    return (((1, 2, 3), (4,)), ((2, 3, 4), (5,)))


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 2, 32, 32, 16, 1, _rolling_tiny(), 1, None, 1e-3, 0.9, 2.0, "f32",
                     description="H=2 hd=32 d=64, frame 32 tokens, sink 16, rolling 3-frame history, "
                                 "2 chunks of 1 frame (64 rows), fp32"),
    "l1_3b": Workload("l1_3b", 12, 128, 1560, 1560, 3, _single_chunk(9, 3), 1, None, 1e-2, 0.9, 2.0, "bf16",
                      description="one Wan/LongLive-1.3B-like layer: d=1536 H=12 hd=128, chunk 4680 queries, "
                                  "sink 1560, history 9 frames (14040 keys), bf16"),
    "warm30": Workload("warm30", 12, 128, 1560, 1560, 3, _warmup_chunks(4, 3), 30, 15, 1e-2, 0.9, 2.0, "bf16",
                       per_layer_scale=True,
                       description="30-layer 1.3B-like warmup: 4 chunks of 3 frames, history 0->9 frames, "
                                   "K=15 L-Layers, bf16 activations, fp32 stats"),
    "l14b": Workload("l14b", 40, 128, 1560, 1560, 3, _warmup_chunks(4, 3), 40, 20, 1e-2, 0.9, 2.0, "bf16",
                     per_layer_scale=True,
                     description="14B-like (Krea-Realtime shape): d=5120 H=40 hd=128, 40 layers, same token "
                                 "geometry, K=20"),
}

LONGHIST_FRAMES = (3, 15, 30, 60, 120)


def longhist(hist_frames: int) -> Workload:
    """Long-history stress shape: one 1.3B-like layer, history of `hist_frames` latent frames, rho=0.95."""
    return Workload(f"longhist{hist_frames}", 12, 128, 1560, 1560, 3, _single_chunk(hist_frames, 3), 1, None,
                    None, 0.95, 2.0, "bf16",
                    description=f"long-history stress: d=1536, 4680 queries, history {hist_frames} frames "
                                f"({hist_frames * 1560} keys), rho=0.95, bf16")


def get_workload(name: str) -> Workload:
    if name.startswith("longhist"):
        return longhist(int(name[len("longhist"):]))
    return WORKLOADS[name]


def scaled(wl: Workload, **kw) -> Workload:
    """A copy of a workload with some fields replaced (used for reduced-size test variants)."""
    return dataclasses.replace(wl, **kw)


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(k) for k in key])))


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32 holding bf16 values."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    b = x.view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32)


def _store(wl: Workload, x: np.ndarray) -> np.ndarray:
    x = x.astype(np.float32, copy=False)
    return round_bf16(x) if wl.dtype == "bf16" else x


def kv_timeline(wl: Workload, layer: int, which: str, seed: int = 0, n_frames: Optional[int] = None) -> np.ndarray:
    """The AR(1) K or V timeline of one layer: float32 [n_frames, frame_tokens, H, hd] (unrounded)."""
    tid = _T_K if which == "k" else _T_V
    rng = _rng(seed, layer, 0, tid)
    F = wl.n_frames if n_frames is None else n_frames
    shape = (wl.frame_tokens, wl.n_heads, wl.head_dim)
    out = np.empty((F,) + shape, dtype=np.float32)
    out[0] = rng.standard_normal(shape, dtype=np.float32)
    a = np.float32(wl.rho)
    b = np.float32(np.sqrt(1.0 - wl.rho * wl.rho))
    for f in range(1, F):
        out[f] = a * out[f - 1] + b * rng.standard_normal(shape, dtype=np.float32)
    return out


def logit_scale(wl: Workload, layer: int, seed: int = 0) -> float:
    if not wl.per_layer_scale or wl.n_layers < 2:
        return wl.logit_std
    perm = _rng(seed, 0, 0, _T_PERM).permutation(wl.n_layers)
    return wl.logit_std * (0.75 + 0.5 * float(perm[layer]) / (wl.n_layers - 1))


def attention_inputs(wl: Workload, layer: int = 0, chunk: int = 0, seed: int = 0,
                     timelines: Optional[tuple] = None) -> Dict[str, np.ndarray]:
    """Q and the three K/V segments of one (layer, chunk) call.

    Returns float32 arrays, each [tokens, H, hd]: q, k_sink, v_sink, k_loc, v_loc, k_hist, v_hist.
    `timelines` may pass precomputed (K, V) timelines of this layer to avoid regenerating them.
    """
    hist_frames, cur_frames = wl.chunks[chunk]
    if timelines is None:
        timelines = (kv_timeline(wl, layer, "k", seed), kv_timeline(wl, layer, "v", seed))
    out = {}
    for name, tl in (("k", timelines[0]), ("v", timelines[1])):
        out[name + "_sink"] = _store(wl, tl[0, : wl.n_sink])
        out[name + "_loc"] = _store(wl, tl[list(cur_frames)].reshape(-1, wl.n_heads, wl.head_dim))
        if hist_frames:
            out[name + "_hist"] = _store(wl, tl[list(hist_frames)].reshape(-1, wl.n_heads, wl.head_dim))
        else:
            out[name + "_hist"] = np.zeros((0, wl.n_heads, wl.head_dim), dtype=np.float32)
    rng = _rng(seed, layer, chunk, _T_Q)
    nq = len(cur_frames) * wl.frame_tokens
    q = rng.standard_normal((nq, wl.n_heads, wl.head_dim), dtype=np.float32) * np.float32(logit_scale(wl, layer, seed))
    out["q"] = _store(wl, q)
    return out


def weight(wl: Workload, layer: int = 0, seed: int = 0) -> np.ndarray:
    """Output-projection weight W of one layer, float32 [d_in, d_out] (y = x @ W), N(0, 1/d)."""
    rng = _rng(seed, layer, 0, _T_W)
    w = rng.standard_normal((wl.d, wl.d), dtype=np.float32) * np.float32(1.0 / np.sqrt(wl.d))
    return _store(wl, w)


def sample_rows(n_rows: int, n_sample: int, seed: int = 0, salt: int = 0) -> np.ndarray:
    """A seeded sorted sample of distinct row indices in [0, n_rows); always includes the last row."""
    if n_sample >= n_rows:
        return np.arange(n_rows)
    rng = _rng(seed, salt, 0, _T_ROWS)
    idx = rng.choice(n_rows - 1, size=n_sample - 1, replace=False)
    return np.sort(np.concatenate([idx, [n_rows - 1]]))


def gaussian(shape: Sequence[int], seed: int, salt: int = 0, scale: float = 1.0) -> np.ndarray:
    """Plain seeded N(0, scale^2) float64 array (for invariant and planted-structure tests)."""
    return _rng(seed, salt, 7, 11).standard_normal(tuple(shape)) * scale
