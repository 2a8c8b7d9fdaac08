"""The per-chunk warmup loop of one layer (ISPA summary, section 2, stage 1: dual-stream attention and
the statistics of every warmup chunk) replayed from a captured CUDA graph gives the eager results."""
import numpy as np
import pytest

import ispa_inputs as inp
from gpu_helpers import host

pytestmark = pytest.mark.gpu


def test_graph_replay_matches_eager(cuda_ok):
    import torch
    from kv_cache_compression_tma_b200.warmup import LayerWarmup
    wl = inp.Workload("graph", 2, 128, 100, 40, 3, inp._warmup_chunks(3, 3), 1, None, 1e-2, 0.9, 2.0, "bf16")
    w = LayerWarmup(wl.n_heads, wl.head_dim, wl.frame_tokens, wl.n_sink, wl.chunks, wl.n_frames)
    k = inp.round_bf16(inp.kv_timeline(wl, 0, "k"))
    v = inp.round_bf16(inp.kv_timeline(wl, 0, "v"))
    w.k.copy_(torch.from_numpy(k))
    w.v.copy_(torch.from_numpy(v))
    for c in range(len(wl.chunks)):
        x = inp.attention_inputs(wl, 0, c, timelines=(k, v))
        w.q[c].copy_(torch.from_numpy(x["q"]))
    w.launch()
    torch.cuda.synchronize()
    eager = [host(t).copy() for t in w.GRS] + [host(w.o_loc).copy(), host(w.dd).copy()]
    for t in w.GRS + [w.o_loc, w.dd]:
        t.zero_()
    w.capture()
    for t in w.GRS + [w.o_loc, w.dd]:
        t.zero_()
    for _ in range(2):
        w.run()
    torch.cuda.synchronize()
    got = [host(t) for t in w.GRS] + [host(w.o_loc), host(w.dd)]
    for a, b in zip(got, eager):
        assert np.array_equal(a, b)   # one row range per statistics block at this width: deterministic
    from kv_cache_compression_tma_b200 import ispa
    assert ispa.get_device_status() == ispa.ISPA_OK
