"""The warmup of one layer (ISPA summary, section 2, stage 1): for every warmup chunk, the dual-stream
attention pass and the statistics update G, R, S -- optionally captured once into a CUDA graph and
replayed, so that the per-chunk launches cost one graph launch per layer.

Orchestration only: every step runs in libispa's kernels (ispa_dual_stream_attn, ispa_accum_stats).
A graph binds the buffers it was captured with (tensor maps and pointers are baked into its kernel
parameters), so the inputs are copied into this object's buffers (or written there by the caller)
before each replay.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

from . import ispa


class LayerWarmup:
    """Buffers and launch sequence of one layer's warmup chunks.

    chunks: per chunk (n_q, n_sink, n_local, n_hist); every chunk's K/V segments are views into one
    K and one V timeline of `n_frames` x `frame_tokens` tokens (sink = the first n_sink tokens of
    frame 0, local = the chunk's frames, history = the frames in between), as in a streaming
    generator's cache.
    """

    def __init__(self, n_heads: int, head_dim: int, frame_tokens: int, n_sink: int,
                 chunk_frames: Sequence[Tuple[Sequence[int], Sequence[int]]], n_frames: int, dtype=None,
                 device="cuda"):
        import torch
        dtype = dtype or torch.bfloat16
        self.H, self.hd, self.F, self.n_sink = n_heads, head_dim, frame_tokens, n_sink
        self.chunks = [(tuple(h), tuple(c)) for h, c in chunk_frames]
        d = n_heads * head_dim
        self.k = torch.zeros((n_frames, frame_tokens, n_heads, head_dim), dtype=dtype, device=device)
        self.v = torch.zeros_like(self.k)
        self.q: List = [torch.zeros((len(c) * frame_tokens, n_heads, head_dim), dtype=dtype, device=device)
                        for _, c in self.chunks]
        nq = max(q.shape[0] for q in self.q)
        self.o_loc = torch.empty((nq, d), dtype=dtype, device=device)
        self.o_full = torch.empty_like(self.o_loc)
        self.dd = torch.empty_like(self.o_loc)
        self.lse_loc = torch.empty((n_heads, nq), dtype=torch.float32, device=device)
        self.lse_hist = torch.empty_like(self.lse_loc)
        self.GRS = [torch.empty((d, d), dtype=torch.float32, device=device) for _ in range(3)]
        self.graph = None

    def _frames(self, t, fr):
        if not fr:
            return t[0, :0]
        return t[fr[0]:fr[-1] + 1].reshape(-1, self.H, self.hd)

    def launch(self):
        """Enqueue every chunk's attention and statistics on the current stream."""
        for c, (hist, cur) in enumerate(self.chunks):
            n = self.q[c].shape[0]
            ks, vs = self.k[0, :self.n_sink], self.v[0, :self.n_sink]
            ispa.dual_stream_attn(self.q[c], ks, vs, self._frames(self.k, cur), self._frames(self.v, cur),
                                  self._frames(self.k, hist), self._frames(self.v, hist), o_loc=self.o_loc[:n],
                                  o_full=self.o_full[:n], lse_loc=self.lse_loc[:, :n], lse_hist=self.lse_hist[:, :n],
                                  d_out=self.dd[:n])
            ispa.accum_stats(self.o_loc[:n], self.dd[:n], *self.GRS, zero=(c == 0))

    def capture(self):
        """Capture launch() into a CUDA graph (after one eager run, so that one-time set-up such as
        the library's device-address lookups happens outside the capture)."""
        import torch
        self.launch()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.launch()
        self.graph = g
        return g

    def run(self):
        """Replay the captured graph if there is one, else launch eagerly."""
        if self.graph is not None:
            self.graph.replay()
        else:
            self.launch()
