"""Benchmark of the ISPA hot path on B200 (one JSON line on stdout from rank 0).

One step = one pass of the whole hot path over one layer's warmup, by default on the 14B-like layer
(Krea-Realtime shape: d = 5120, 40 heads x 128; latent frames of 1560 tokens, 3-frame chunks of 4680
queries, a 1-frame sink, history growing 0 -> 3 -> 6 -> 9 frames over the four warmup chunks):
  1. per warmup chunk: decomposable dual-stream attention (A_loc, A_full, lse_loc, lse_hist,
     D = A_full - A_loc in one pass) and the statistics G, R, S accumulated from A_loc and D,
  2. at T_warm: the closed-form ridge absorb dW = (G + lam I)^-1 R W with lam = 1e-2 tr(G)/d, the
     reconstruction error eps and eps_rel, and W_new = W + dW,
  3. the layer selection on the host from the eps read back.
value = query tokens per second of the whole step (all ranks).  Multi-GPU runs are replicas: each
rank processes its own independent layer, no collective on the data path (weak scaling).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]
                  [--stack] [--infer] [--overhead]

--workload: l14b (default), l1_3b (one 9-frame-history chunk of the 1.3B-like layer), warm30 (one
layer of the 1.3B-like warmup), longhistN (one 1.3B-like chunk with N history frames), tiny.
--stack: time the whole multi-layer warmup of warm30 / l14b (every layer's chunks, every absorb and
the selection) instead of one layer.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import ispa_inputs as inp  # noqa: E402

METRIC = "dual-stream attn TFLOP/s (% bf16 peak) + absorb ms/layer; query tokens/s"
UNIT = "query tok/s"
L2_FLUSH_BYTES = 256 << 20
DEFAULT_WORKLOAD = "l14b"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def peak_source(peaks):
    if peaks["source"] == "measured":
        return "measured bf16 matmul burst (MEASURED_PEAKS.json)"
    return "fallback bf16 matmul burst of the profiling recipe (MEASURED_PEAKS.json absent)"


def n_keys(wl, c):
    return wl.n_sink + wl.n_local(c) + wl.n_hist(c)


def workload_config(wl):
    C = len(wl.chunks)
    return {"workload": f"{wl.name}: {wl.description}", "chunks": C,
            "n_q_per_chunk": [wl.n_q(c) for c in range(C)],
            "n_kv_per_chunk": [[wl.n_sink, wl.n_local(c), wl.n_hist(c)] for c in range(C)],
            "d": wl.d, "heads": wl.n_heads, "head_dim": wl.head_dim, "lam_rel": wl.lam_rel or 1e-2,
            "l2": "flushed between timed steps (256 MiB write, outside the timed events); the layer's "
                  "K/V cache alone exceeds L2 on the 14B-like layer",
            "parallelism": "replicas (one independent layer per rank)"}


def attn_flops(wl, c):
    """Algorithmic FLOPs of one dual-stream launch: QK^T and PV over every key once, all heads."""
    return 4.0 * wl.n_q(c) * n_keys(wl, c) * wl.d


def stats_flops(wl, c):
    """Algorithmic FLOPs of one statistics launch: G and S are symmetric (one triangle each) and R is
    a full product, i.e. 2 + 2 = 4 n_q d^2 (a full Gram is 2 n_q d^2)."""
    return 4.0 * wl.n_q(c) * wl.d * wl.d


def absorb_flops(d):
    """Algorithmic FLOPs of the absorb: R W and S W (2 d^3 each), Cholesky (d^3 / 3), and the two
    triangular solves with d right-hand sides (d^3 each): about 6.33 d^3."""
    return (2.0 + 2.0 + 1.0 / 3.0 + 2.0) * d ** 3


# --------------------------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        return summarize_clocks(self.lines)


def summarize_clocks(lines):
    """Median SM clock under load, the maximum, and every throttle reason seen active."""
    mhz, mx, reasons, power = [], None, set(), []
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for ln in lines:
        parts = [p.strip() for p in ln.split(",")]
        if len(parts) < 9:
            continue
        try:
            mhz.append(float(parts[1]))
            mx = float(parts[2])
            power.append(float(parts[3]))
        except ValueError:
            continue
        for name, val in zip(names, parts[5:9]):
            if val.lower() == "active":
                reasons.add(name)
    under_load = [m for m in mhz if m > 500] or mhz
    return {"sm_mhz": float(np.median(under_load)) if under_load else None, "sm_max_mhz": mx,
            "reasons": sorted(reasons), "samples": len(mhz),
            "power_w_median": float(np.median(power)) if power else None}


def attn_traffic(workload):
    """DRAM bytes per attention launch from the committed ncu capture, or None when the capture was of
    another workload or the kernel source has changed since the counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"attn_tc_{workload}.json")
    src = os.path.join(ROOT, "kv_cache_compression_tma_b200", "csrc", "attn_tc.cu")
    try:
        tj = json.load(open(path))
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if tj.get("workload") == workload and tj.get("kernel_src_sha256_16") == sha:
            return tj.get("bytes_per_launch")
    except Exception:
        pass
    return None


# --------------------------------------------------------------------------------------------- inputs
def gpu_inputs(wl, layer, seed, torch):
    """The input recipe of ispa_inputs drawn on the GPU (seeded torch generator): AR(1) K/V timelines
    across latent frames, Gaussian Q per chunk scaled to the layer's logit std, W ~ N(0, 1/d); all
    rounded to bf16.  Returns (K timeline, V timeline, [Q per chunk], W), timelines [F, T, H, hd]."""
    g = torch.Generator(device="cuda")
    g.manual_seed((seed * 1000003 + layer) & 0x7FFFFFFF)
    shape = (wl.n_frames, wl.frame_tokens, wl.n_heads, wl.head_dim)
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    tl = []
    for _ in range(2):
        x = torch.empty(shape, dtype=torch.float32, device="cuda")
        x[0].normal_(generator=g)
        a, b = wl.rho, math.sqrt(1.0 - wl.rho * wl.rho)
        for f in range(1, wl.n_frames):
            x[f].normal_(generator=g).mul_(b).add_(x[f - 1], alpha=a)
        tl.append(x.to(dt))
        del x
    s = inp.logit_scale(wl, layer, seed)
    qs = [(torch.randn((wl.n_q(c), wl.n_heads, wl.head_dim), generator=g, device="cuda") * s).to(dt)
          for c in range(len(wl.chunks))]
    W = (torch.randn((wl.d, wl.d), generator=g, device="cuda") / math.sqrt(wl.d)).to(dt)
    return tl[0], tl[1], qs, W


def segments(wl, k_tl, v_tl, c):
    """((k_sink, k_loc, k_hist), (v_sink, v_loc, v_hist)) of chunk c as views into the timelines."""
    hist, cur = wl.chunks[c]

    def frames(t, fr):
        if not fr:
            return t[0, :0]
        return t[fr[0]:fr[-1] + 1].reshape(-1, wl.n_heads, wl.head_dim)
    return [(t[0, :wl.n_sink], frames(t, cur), frames(t, hist)) for t in (k_tl, v_tl)]


# --------------------------------------------------------------------------------------------- GPU arm
class LayerStep:
    """Device buffers and the launch sequence of one step: every warmup chunk of one layer (attention +
    statistics), then the absorb with eps and W_new."""

    def __init__(self, wl, layer, seed, torch, ispa):
        self.torch, self.ispa, self.wl = torch, ispa, wl
        dev = "cuda"
        k_tl, v_tl, qs, W = gpu_inputs(wl, layer, seed, torch)
        self.inputs = [k_tl, v_tl, W] + qs            # one step's input tensors (device)
        C = len(wl.chunks)
        nq_max = max(wl.n_q(c) for c in range(C))
        d, H = wl.d, wl.n_heads
        dt = k_tl.dtype
        self.o_loc = torch.empty((nq_max, d), dtype=dt, device=dev)
        self.o_full = torch.empty_like(self.o_loc)
        self.dd = torch.empty_like(self.o_loc)
        self.lse_loc = torch.empty((H, nq_max), dtype=torch.float32, device=dev)
        self.lse_hist = torch.empty_like(self.lse_loc)
        self.GRS = [torch.empty((d, d), dtype=torch.float32, device=dev) for _ in range(3)]
        self.dW = torch.empty((d, d), dtype=torch.float32, device=dev)
        self.eps = torch.empty((4,), dtype=torch.float64, device=dev)
        self.w_new = torch.empty_like(W)
        self.ws = torch.empty((ispa.absorb_workspace_size(d),), dtype=torch.uint8, device=dev)
        self.eps_host = torch.empty((4,), dtype=torch.float64).pin_memory()
        self.lam_rel = wl.lam_rel or 1e-2
        self.n_events = 2 * C + 2

    def run(self, inputs=None, ev=None):
        """Launch one step on the current stream.  `ev` (2 C + 2 events): start, then after each
        chunk's attention and statistics, then after the absorb."""
        wl, ispa = self.wl, self.ispa
        k_tl, v_tl, W, *qs = inputs or self.inputs
        if ev:
            ev[0].record()
        for c in range(len(wl.chunks)):
            (ks, kl, kh), (vs, vl, vh) = segments(wl, k_tl, v_tl, c)
            n = wl.n_q(c)
            ispa.dual_stream_attn(qs[c], ks, vs, kl, vl, kh, vh, o_loc=self.o_loc[:n], o_full=self.o_full[:n],
                                  lse_loc=self.lse_loc[:, :n], lse_hist=self.lse_hist[:, :n], d_out=self.dd[:n])
            if ev:
                ev[1 + 2 * c].record()
            ispa.accum_stats(self.o_loc[:n], self.dd[:n], *self.GRS, zero=(c == 0))
            if ev:
                ev[2 + 2 * c].record()
        ispa.absorb(*self.GRS, W, self.lam_rel, lam_rel=True, dW=self.dW, eps=self.eps, w_new=self.w_new,
                    write_wnew=True, ws=self.ws)
        if ev:
            ev[-1].record()

    def finish_host(self):
        """Host side of the step: the selection over this rank's layer from the eps read back."""
        idx, mask, st = self.ispa.select_layers([float(self.eps_host[0])], 1)
        return idx


class E2E:
    """The same step through the public API from pinned host buffers, double-buffered: step i+1's
    inputs cross PCIe on a copy stream (one cudaMemcpyAsync per tensor) while step i computes; each
    step ends with the D2H read of its eps (the selection's input) into pinned memory."""

    def __init__(self, step, torch):
        self.step, self.torch = step, torch
        self.host = [t.cpu().pin_memory() for t in step.inputs]
        self.bufs = [step.inputs, [torch.empty_like(t) for t in step.inputs]]
        self.copy_stream = torch.cuda.Stream()
        self.h2d_bytes = sum(t.numel() * t.element_size() for t in self.host)
        self.d2h_bytes = step.eps_host.numel() * step.eps_host.element_size()

    def run(self, K):
        torch = self.torch
        comp = torch.cuda.current_stream()
        copied = [torch.cuda.Event() for _ in range(K)]
        done = [torch.cuda.Event() for _ in range(K)]
        start = torch.cuda.Event()
        start.record(comp)

        def h2d(i):
            with torch.cuda.stream(self.copy_stream):
                self.copy_stream.wait_event(start)
                if i >= 2:
                    self.copy_stream.wait_event(done[i - 2])  # buffer set i % 2 is free again
                for dst, src in zip(self.bufs[i % 2], self.host):
                    dst.copy_(src, non_blocking=True)
                copied[i].record(self.copy_stream)

        h2d(0)
        for i in range(K):
            if i + 1 < K:
                h2d(i + 1)
            comp.wait_event(copied[i])
            self.step.run(inputs=self.bufs[i % 2])
            self.step.eps_host.copy_(self.step.eps, non_blocking=True)
            done[i].record(comp)


def max_over_ranks(values, world, device):
    """Each timing is the maximum over the ranks (one all-reduce; with one rank, the values as given)."""
    import torch
    vals = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(vals, op=dist.ReduceOp.MAX)
    return [float(v) for v in vals.cpu()]


def aggregate_value(world, n_q, steps, total_ms):
    """Whole-job throughput: every rank processes its own layer (replicas), so query tokens of all
    ranks over the slowest rank's time."""
    return world * n_q * steps / (total_ms / 1e3)


def gpu_arm(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import kv_cache_compression_tma_b200 as ispa

    torch.cuda.set_device(local_rank)
    wl = inp.get_workload(args.workload)
    C = len(wl.chunks)
    step = LayerStep(wl, layer=rank, seed=args.seed, torch=torch, ispa=ispa)
    flush = torch.empty((L2_FLUSH_BYTES // 4,), dtype=torch.float32, device="cuda")
    K, W = args.steps, args.warmup

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(W):
        flush.fill_(1.0)
        step.run()
    torch.cuda.synchronize()
    st = ispa.get_device_status()
    if st != 0:
        raise RuntimeError("device status after warm-up: " + ispa.status_string(st))

    # ---- timed region: K steps, each bracketed by events; L2 flushed between steps, outside the events
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(step.n_events)] for _ in range(K)]
    sampler = ClockSampler(local_rank).start()
    launches0 = ispa.launch_count()
    barrier()
    torch.cuda.synchronize()
    for i in range(K):
        flush.fill_(1.0)
        step.run(ev=evs[i])
    torch.cuda.synchronize()
    barrier()
    launches = ispa.launch_count() - launches0
    clocks = sampler.stop()
    st = ispa.get_device_status()
    if st != 0:
        raise RuntimeError("device status after timed steps: " + ispa.status_string(st))
    step_ms = [e[0].elapsed_time(e[-1]) for e in evs]
    attn_ms = [[e[2 * c].elapsed_time(e[1 + 2 * c]) for e in evs] for c in range(C)]
    stats_ms = [[e[1 + 2 * c].elapsed_time(e[2 + 2 * c]) for e in evs] for c in range(C)]
    absorb_ms = [e[-2].elapsed_time(e[-1]) for e in evs]
    step.eps_host.copy_(step.eps)
    host_sel = step.finish_host()

    # ---- end to end through the public API with host buffers (H2D inputs, D2H eps), double-buffered
    e2e = E2E(step, torch)
    e2e.run(max(1, W))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record()
    e2e.run(K)
    e1.record()
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1) / K
    step.finish_host()
    st = ispa.get_device_status()
    if st != 0:
        raise RuntimeError("device status after the end-to-end steps: " + ispa.status_string(st))

    total_ms = float(sum(step_ms))
    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], world, "cuda")
    if rank != 0:
        return None
    peaks = load_peaks()
    rows = wl.rows_per_layer
    ms_per_step = total_ms / K
    value = aggregate_value(world, rows, K, total_ms)
    cw = C - 1  # the T_warm chunk: the longest history
    attn_avg = [float(np.mean(a)) for a in attn_ms]
    stats_avg = [float(np.mean(s)) for s in stats_ms]
    af = attn_flops(wl, cw)
    achieved = af / (attn_avg[cw] / 1e3) / 1e12
    absorb_avg = float(np.mean(absorb_ms))
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if wl.dtype == "bf16" else "f32",
        "data": "synthetic: seeded AR(1) K/V across latent frames, Gaussian Q and W (the ispa_inputs recipe, "
                "drawn on the GPU)",
        "config": workload_config(wl),
        "roofline": {"bound": "tensor", "kernel": "attn_tc_kernel<128> (T_warm chunk)", "achieved": achieved,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                     "peak_source": peak_source(peaks), "frac_of": peaks["source"],
                     "algorithmic_flops_per_launch": af, "traffic": attn_traffic(wl.name)},
        "attn_ms_per_chunk": attn_avg,
        "attn_tflops_per_chunk": [attn_flops(wl, c) / (attn_avg[c] / 1e3) / 1e12 for c in range(C)],
        "attn_frac_bf16_peak_t_warm": achieved / peaks["bf16_tflops"],
        "stats_ms_per_chunk": stats_avg,
        "stats_tflops_algorithmic": [stats_flops(wl, c) / (stats_avg[c] / 1e3) / 1e12 for c in range(C)],
        "absorb_ms_per_layer": absorb_avg,
        "absorb_tflops_algorithmic": absorb_flops(wl.d) / (absorb_avg / 1e3) / 1e12,
        "gram_plus_absorb_ms": stats_avg[cw] + absorb_avg,
        "all_chunks_gram_plus_absorb_ms": float(sum(stats_avg)) + absorb_avg,
        "e2e": {"value": world * rows / (e2e_ms / 1e3), "unit": UNIT, "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": e2e.h2d_bytes, "d2h_bytes_per_step": e2e.d2h_bytes,
                "overlap": "double-buffered: step i+1's H2D on a copy stream during step i"},
        "gpu_launches": int(launches),
        "gpu_launches_per_step": launches / K,
        "clocks": clocks,
        "selected": [int(i) for i in host_sel],
    }
    if not args.no_cpu_baseline and world == 1:
        host_in = [t.float().cpu().numpy() for t in step.inputs]
        line["cpu_baseline"] = cpu_baseline(wl, host_in, args.seed, n_sample=args.cpu_rows)
    return line


def time_interleaved(fns, steps, warmup, flush, torch):
    """CUDA-event times of each (name, fn) of `fns`: every function is warmed up, then each of the
    `steps` rounds runs all of them once, starting one further along the list each round, so that a
    clock that drifts during the run (the power cap) weighs on every function alike.  L2 is flushed
    before every timed call, outside the events.  Returns {name: [ms per call]}."""
    for _, fn in fns:
        for _ in range(warmup):
            fn()
    ms = {name: [] for name, _ in fns}
    for i in range(steps):
        k = i % len(fns)
        for name, fn in fns[k:] + fns[:k]:
            flush.fill_(1.0)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ms[name].append(e0.elapsed_time(e1))
    return ms


# --------------------------------------------------------------------------------------------- multi-layer warmups
def overhead_arm(args):
    """Cost of collecting both streams (the pages call it negligible): on the T_warm chunk of one layer
    of the workload, plain single-branch attention over every key (sink and history in one segment,
    so the kernel keeps one softmax state) against the dual-stream pass, the dual-stream pass with D,
    and the dual-stream pass with D plus the Gram statistics.  CUDA events, L2 flushed between
    repetitions, the modes taking turns (`time_interleaved`), medians."""
    import torch
    import kv_cache_compression_tma_b200 as ispa
    wl = inp.get_workload(args.workload)
    step = LayerStep(wl, layer=0, seed=args.seed, torch=torch, ispa=ispa)
    k_tl, v_tl, W, *qs = step.inputs
    c = len(wl.chunks) - 1
    (ks, kl, kh), (vs, vl, vh) = segments(wl, k_tl, v_tl, c)
    q = qs[c]
    n = wl.n_q(c)
    one = torch.cat([ks, kh], 0), torch.cat([vs, vh], 0)
    flush = torch.empty((L2_FLUSH_BYTES // 4,), dtype=torch.float32, device="cuda")
    out = dict(o_loc=step.o_loc[:n], o_full=step.o_full[:n], lse_loc=step.lse_loc[:, :n], lse_hist=step.lse_hist[:, :n])

    def plain():
        ispa.dual_stream_attn(q, one[0], one[1], kl, vl, kl[:0], vl[:0], want_delta=False, **out)

    def dual():
        ispa.dual_stream_attn(q, ks, vs, kl, vl, kh, vh, want_delta=False, **out)

    def dual_d():
        ispa.dual_stream_attn(q, ks, vs, kl, vl, kh, vh, d_out=step.dd[:n], **out)

    def dual_d_stats():  # the T_warm chunk accumulates into the layer's statistics
        dual_d()
        ispa.accum_stats(step.o_loc[:n], step.dd[:n], *step.GRS, zero=False)

    # the whole per-chunk warmup loop of the layer, eager and replayed from a CUDA graph
    from kv_cache_compression_tma_b200.warmup import LayerWarmup
    lw = LayerWarmup(wl.n_heads, wl.head_dim, wl.frame_tokens, wl.n_sink, wl.chunks, wl.n_frames)
    lw.k.copy_(k_tl)
    lw.v.copy_(v_tl)
    for c in range(len(wl.chunks)):
        lw.q[c].copy_(qs[c])

    def warmup_eager():
        lw.launch()

    def warmup_graph():
        if lw.graph is None:  # captured during the untimed warm-up calls
            lw.capture()
        lw.run()

    sampler = ClockSampler(0).start()
    fns = [("plain_attention", plain), ("dual_stream", dual), ("dual_stream_with_d", dual_d),
           ("dual_stream_with_d_and_stats", dual_d_stats), ("layer_warmup_eager", warmup_eager),
           ("layer_warmup_graph", warmup_graph)]
    times = time_interleaved(fns, args.steps, args.warmup, flush, torch)
    res = {name + "_ms": float(np.median(v)) for name, v in times.items()}
    clocks = sampler.stop()
    if ispa.get_device_status() != 0:
        raise RuntimeError("device status after the overhead runs")
    base = res["plain_attention_ms"]
    for name in ("dual_stream", "dual_stream_with_d", "dual_stream_with_d_and_stats"):
        res[name + "_overhead"] = res[name + "_ms"] / base - 1.0
    res["layer_warmup_graph_speedup"] = res["layer_warmup_eager_ms"] / res["layer_warmup_graph_ms"]
    return {"mode": "collection_overhead", "workload": wl.name, "chunk": c, "steps": args.steps,
            "warmup": args.warmup, "clocks": clocks, **res}


def history_sweep_arm(args):
    """Long-history stress: one 1.3B-like chunk (4680 queries, 1560-token sink, 3-frame local chunk)
    with N history frames, N in 3, 15, 30, 60, 120 (up to 187,200 keys, rho = 0.95 across frames):
    dual-stream attention time, TFLOP/s and its fraction of the bf16 peak, and the HBM rate of the
    algorithmic bytes (Q, K/V once, O_loc, O_full, D, lse) against the copy peak.  CUDA events, L2
    flushed between repetitions."""
    import torch
    import kv_cache_compression_tma_b200 as ispa
    peaks = load_peaks()
    flush = torch.empty((L2_FLUSH_BYTES // 4,), dtype=torch.float32, device="cuda")
    rows = []
    sampler = ClockSampler(0).start()
    for nh in (3, 15, 30, 60, 120):
        wl = inp.get_workload(f"longhist{nh}")
        k_tl, v_tl, qs, W = gpu_inputs(wl, 0, args.seed, torch)
        c = len(wl.chunks) - 1
        (ks, kl, kh), (vs, vl, vh) = segments(wl, k_tl, v_tl, c)
        q = qs[c]
        n, d = wl.n_q(c), wl.d
        out = ispa.dual_stream_attn(q, ks, vs, kl, vl, kh, vh)
        kw = dict(o_loc=out["o_loc"], o_full=out["o_full"], lse_loc=out["lse_loc"], lse_hist=out["lse_hist"],
                  d_out=out["d"])
        for _ in range(args.warmup):
            ispa.dual_stream_attn(q, ks, vs, kl, vl, kh, vh, **kw)
        ms = []
        for _ in range(args.steps):
            flush.fill_(1.0)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            ispa.dual_stream_attn(q, ks, vs, kl, vl, kh, vh, **kw)
            e1.record()
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        t = float(np.mean(ms))
        nk = n_keys(wl, c)
        flops = attn_flops(wl, c)
        nbytes = 2 * n * d + 2 * 2 * nk * d + 3 * 2 * n * d + 2 * 4 * wl.n_heads * n
        rows.append({"history_frames": nh, "keys": nk, "ms": t, "tflops": flops / (t / 1e3) / 1e12,
                     "frac_bf16_peak": flops / (t / 1e3) / 1e12 / peaks["bf16_tflops"],
                     "algorithmic_bytes": nbytes, "hbm_gbs": nbytes / (t / 1e3) / 1e9,
                     "frac_hbm_peak": nbytes / (t / 1e3) / 1e9 / peaks["hbm_gbs"]})
        del k_tl, v_tl, qs, W, out, kw, ks, kl, kh, vs, vl, vh, q
        torch.cuda.empty_cache()
    clocks = sampler.stop()
    if ispa.get_device_status() != 0:
        raise RuntimeError("device status after the history sweep")
    return {"mode": "history_sweep", "workload": "longhistN: one 1.3B-like chunk, d=1536 H=12 hd=128, bf16",
            "peak_source": peak_source(peaks), "hbm_peak_gbs": peaks["hbm_gbs"], "steps": args.steps,
            "warmup": args.warmup, "clocks": clocks, "rows": rows}


def warmup_arm(args):
    """Timing of a whole multi-layer warmup: per layer, every chunk's dual-stream attention and
    statistics, then the absorb of every layer and the selection of the K lowest-eps layers."""
    import torch
    import kv_cache_compression_tma_b200 as ispa
    wl = inp.get_workload(args.workload)
    L = min(wl.n_layers, args.layers or wl.n_layers)
    d, H = wl.d, wl.n_heads
    layers = [gpu_inputs(wl, l, args.seed, torch) for l in range(L)]
    stats = [[torch.empty((d, d), dtype=torch.float32, device="cuda") for _ in range(3)] for _ in range(L)]
    nq_max = max(wl.n_q(c) for c in range(len(wl.chunks)))
    o_loc = torch.empty((nq_max, d), dtype=torch.bfloat16, device="cuda")
    o_full, dd = torch.empty_like(o_loc), torch.empty_like(o_loc)
    lse_l = torch.empty((H, nq_max), dtype=torch.float32, device="cuda")
    lse_h = torch.empty_like(lse_l)
    dW = torch.empty((d, d), dtype=torch.float32, device="cuda")
    eps = torch.empty((L, 4), dtype=torch.float64, device="cuda")
    ws = torch.empty((ispa.absorb_workspace_size(d),), dtype=torch.uint8, device="cuda")
    w_new = [torch.empty_like(layers[l][3]) for l in range(L)]
    k_sel = (wl.k_select or max(1, L // 2)) if L == wl.n_layers else max(1, L // 2)

    def run(ev=None):
        for l in range(L):
            k_tl, v_tl, qs, W = layers[l]
            for c in range(len(wl.chunks)):
                (ks, kl, kh), (vs, vl, vh) = segments(wl, k_tl, v_tl, c)
                n = wl.n_q(c)
                ispa.dual_stream_attn(qs[c], ks, vs, kl, vl, kh, vh, o_loc=o_loc[:n], o_full=o_full[:n],
                                      lse_loc=lse_l[:, :n], lse_hist=lse_h[:, :n], d_out=dd[:n])
                ispa.accum_stats(o_loc[:n], dd[:n], *stats[l], zero=(c == 0))
        if ev:
            ev[1].record()
        for l in range(L):
            ispa.absorb(*stats[l], layers[l][3], wl.lam_rel, lam_rel=True, dW=dW, eps=eps[l], w_new=w_new[l],
                        write_wnew=True, ws=ws)
        if ev:
            ev[2].record()
        e = eps[:, 0].cpu().numpy()
        return ispa.select_layers(e, k_sel)

    # Pipelined form of the same work: the statistics of a chunk run on a side stream while the next
    # chunk's attention runs (two output buffer sets), and each layer's absorb starts on a third
    # stream as soon as that layer's statistics are complete, under the later layers' attention.
    s_stats, s_abs = torch.cuda.Stream(), torch.cuda.Stream()
    bufs = [(o_loc, o_full, dd, lse_l, lse_h),
            tuple(torch.empty_like(t) for t in (o_loc, o_full, dd, lse_l, lse_h))]
    ev_stats = [torch.cuda.Event(), torch.cuda.Event()]

    def run_overlap(ev=None):
        main = torch.cuda.current_stream()
        i = 0
        for l in range(L):
            k_tl, v_tl, qs, W = layers[l]
            for c in range(len(wl.chunks)):
                b = i % 2
                ol, of, dl, ll, lh = bufs[b]
                (ks, kl, kh), (vs, vl, vh) = segments(wl, k_tl, v_tl, c)
                n = wl.n_q(c)
                if i >= 2:
                    main.wait_event(ev_stats[b])  # the statistics of chunk i-2 have read buffer b
                ispa.dual_stream_attn(qs[c], ks, vs, kl, vl, kh, vh, o_loc=ol[:n], o_full=of[:n],
                                      lse_loc=ll[:, :n], lse_hist=lh[:, :n], d_out=dl[:n])
                s_stats.wait_stream(main)
                with torch.cuda.stream(s_stats):
                    ispa.accum_stats(ol[:n], dl[:n], *stats[l], zero=(c == 0))
                    ev_stats[b].record(s_stats)
                i += 1
            s_abs.wait_stream(s_stats)  # layer l's statistics are complete
            with torch.cuda.stream(s_abs):
                ispa.absorb(*stats[l], layers[l][3], wl.lam_rel, lam_rel=True, dW=dW_pipe[l % 2], eps=eps[l],
                            w_new=w_new[l], write_wnew=True, ws=ws)
        if ev:
            ev[1].record()
        main.wait_stream(s_abs)
        main.wait_stream(s_stats)
        if ev:
            ev[2].record()
        e = eps[:, 0].cpu().numpy()
        return ispa.select_layers(e, k_sel)

    dW_pipe = [dW, torch.empty_like(dW)]
    run_fn = run_overlap if args.overlap else run
    for _ in range(max(1, args.warmup)):
        run_fn()
    torch.cuda.synchronize()
    times = []
    sampler = ClockSampler(0).start()
    for _ in range(args.steps):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record()
        idx, mask, st = run_fn(ev)
        torch.cuda.synchronize()
        times.append((ev[0].elapsed_time(ev[1]), ev[1].elapsed_time(ev[2]), ev[0].elapsed_time(ev[2])))
    clocks = sampler.stop()
    if ispa.get_device_status() != 0:
        raise RuntimeError("device status after the warmup runs")
    infer = infer_arm(args, wl, L, layers, w_new, idx, torch) if args.infer else None
    t_attn = float(np.mean([t[0] for t in times]))
    t_abs = float(np.mean([t[1] for t in times]))
    t_all = float(np.mean([t[2] for t in times]))
    rows = wl.rows_per_layer
    flops = sum(attn_flops(wl, c) for c in range(len(wl.chunks)))
    cfg = workload_config(wl)
    cfg.update({"layers_timed": L, "k_select": k_sel, "mode": "stack (pipelined)" if args.overlap else "stack"})
    return {"metric": METRIC, "value": L * rows / (t_all / 1e3), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t_all, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic, drawn on the GPU with the ispa_inputs recipe",
            "config": cfg, "attn_plus_stats_ms": t_attn,
            "attn_stats_tflops": L * flops / (t_attn / 1e3) / 1e12, "absorb_ms_total": t_abs,
            "absorb_ms_per_layer": t_abs / L, "selected": [int(i) for i in idx], "clocks": clocks,
            "note": ("pipelined: statistics overlap the next chunk's attention and each layer's absorb the later "
                     "layers' attention; attn_plus_stats_ms is then the time until the last attention launch "
                     "returns and absorb_ms_total the remaining tail; L2 not flushed between layers")
                    if args.overlap else "attention figures include the statistics GEMMs; L2 not flushed between layers",
            **({"infer": infer} if infer else {})}


def infer_arm(args, wl, L, layers, w_new, idx, torch):
    """One inference chunk after T_warm over the whole stack (T_warm geometry: the last warmup chunk's
    history), timed with every layer an F-Layer and with the selected layers as L-Layers (local-only
    attention, W_new); plus the KV history bytes the L-Layers free."""
    import kv_cache_compression_tma_b200 as ispa
    from kv_cache_compression_tma_b200 import llayer as ll
    c = len(wl.chunks) - 1
    n = wl.n_q(c)
    work = ll.LayerWork(n, wl.n_heads, wl.head_dim, torch.bfloat16)
    y = torch.empty((n, wl.d), dtype=torch.bfloat16, device="cuda")
    sel = set(int(i) for i in idx)

    def step(mixed):
        for l in range(L):
            k_tl, v_tl, qs, W = layers[l]
            (ks, kl, kh), (vs, vl, vh) = segments(wl, k_tl, v_tl, c)
            is_l = mixed and l in sel
            ll.layer_forward(qs[c], ks, vs, kl, vl, kh, vh, w_new[l] if is_l else W, llayer=is_l, work=work, out=y)

    res = {}
    sampler = ClockSampler(0).start()
    for mode in ("all_full", "mixed"):
        for _ in range(max(1, args.warmup)):
            step(mode == "mixed")
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            step(mode == "mixed")
        e1.record()
        torch.cuda.synchronize()
        res["ms_" + mode] = e0.elapsed_time(e1) / args.steps
    # the projection kernel alone (one layer's A [n, d] times W [d, d]) against the bf16 tensor peak
    a = work.o_loc[:n]
    W0 = layers[0][3]
    for _ in range(3):
        ispa.project(a, W0, out=y)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 50
    e0.record()
    for _ in range(reps):
        ispa.project(a, W0, out=y)
    e1.record()
    torch.cuda.synchronize()
    res["clocks"] = sampler.stop()
    proj_ms = e0.elapsed_time(e1) / reps
    peaks = load_peaks()
    peak = peaks["bf16_tflops"]
    proj_tflops = 2.0 * n * wl.d * wl.d / (proj_ms / 1e3) / 1e12
    res.update({"project_ms": proj_ms, "project_tflops": proj_tflops, "project_frac_bf16_peak": proj_tflops / peak})
    # the W8A8 projection of an L-Layer: quantise the activations (per row), fp8 GEMM with the weight
    # quantised once per layer (per output column); the fp8 peak is taken as 2x the measured bf16
    # burst (the nominal dense ratio), not measured
    qw, sw = ispa.quantize_e4m3(W0, columns=True)
    qa, sa = ispa.quantize_e4m3(a)
    for _ in range(3):
        ispa.project_w8a8(qa, sa, qw, sw, out=y)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    ev[0].record()
    for _ in range(reps):
        ispa.quantize_e4m3(a, q=qa, scale=sa)
    ev[1].record()
    for _ in range(reps):
        ispa.project_w8a8(qa, sa, qw, sw, out=y)
    ev[2].record()
    torch.cuda.synchronize()
    q_ms, g_ms = ev[0].elapsed_time(ev[1]) / reps, ev[1].elapsed_time(ev[2]) / reps
    w8_tflops = 2.0 * n * wl.d * wl.d / (g_ms / 1e3) / 1e12
    res.update({"w8a8_quantize_ms": q_ms, "w8a8_gemm_ms": g_ms, "w8a8_gemm_tflops": w8_tflops,
                "w8a8_frac_fp8_peak": w8_tflops / (2.0 * peak),
                "fp8_peak_tflops": 2.0 * peak,
                "fp8_peak_source": f"2 x {peaks['source']} bf16 burst (nominal dense ratio)",
                "w8a8_projection_speedup_vs_bf16": proj_ms / (q_ms + g_ms)})
    if ispa.get_device_status() != 0:
        raise RuntimeError("device status after the inference steps")
    res.update(ll.kv_savings(sel, L, ll.kv_bytes(wl.n_sink, wl.n_local(c), wl.n_hist(c), wl.n_heads, wl.head_dim, 2)))
    res["l_layers"] = len(sel)
    res["query_tok_per_s_mixed"] = L * n / (res["ms_mixed"] / 1e3)
    res["query_tok_per_s_all_full"] = L * n / (res["ms_all_full"] / 1e3)
    return res


def tempcache_arm(args):
    """FAST-AR TempCache on one layer of the workload: the history frames of the T_warm chunk are
    merged frame by frame into a TempCache (threshold args.tc_threshold on the cosine similarity of
    the keys); times the match (tensor-core top-1 over the cache), the merge, and the dual-stream
    attention over the merged history (log-size bias) against the unmerged history."""
    import torch
    import kv_cache_compression_tma_b200 as ispa
    wl = inp.get_workload(args.workload)
    k_tl, v_tl, qs, W = gpu_inputs(wl, 0, args.seed, torch)
    c = len(wl.chunks) - 1
    hist, cur = wl.chunks[c]
    F = wl.frame_tokens
    tc = ispa.TempCache(wl.n_heads, wl.head_dim, capacity=max(1, len(hist)) * F)
    match_ms, merge_ms, cache_len = [], [], []
    for f in hist:
        kf, vf = k_tl[f], v_tl[f]
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record()
        idx, sim = tc.match(kf)
        e[1].record()
        tc.merge(kf, vf, idx, sim, args.tc_threshold)
        e[2].record()
        torch.cuda.synchronize()
        match_ms.append(e[0].elapsed_time(e[1]))
        merge_ms.append(e[1].elapsed_time(e[2]))
        cache_len.append(int(tc.n_valid.max().item()))
    if ispa.get_device_status() != 0:
        raise RuntimeError("device status after the merges")
    n_live = int(tc.n_valid.max().item())
    kh, vh, bias = tc.k[:n_live], tc.v[:n_live], tc.bias[:, :n_live]
    (ks, kl, khu), (vs, vl, vhu) = segments(wl, k_tl, v_tl, c)
    q = qs[c]
    flush = torch.empty((L2_FLUSH_BYTES // 4,), dtype=torch.float32, device="cuda")

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        ms = []
        for _ in range(args.steps):
            flush.fill_(1.0)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        return float(np.mean(ms))

    full_ms = timed(lambda: ispa.dual_stream_attn(q, ks, vs, kl, vl, khu, vhu))
    merged_ms = timed(lambda: ispa.dual_stream_attn(q, ks, vs, kl, vl, kh, vh, kv_bias=(None, None, bias)))
    # match work of the last frame: T new keys against the cache before it, 2 hd flops per pair
    n_prev = cache_len[-2] if len(cache_len) > 1 else 0
    match_flops = 2.0 * F * n_prev * wl.head_dim * wl.n_heads
    return {"mode": "tempcache", "workload": wl.name, "threshold": args.tc_threshold, "history_frames": len(hist),
            "history_tokens": len(hist) * F, "merged_entries_max_head": n_live,
            "kept_fraction": n_live / max(1, len(hist) * F), "entries_after_each_frame": cache_len,
            "match_ms_per_frame": match_ms, "merge_ms_per_frame": merge_ms,
            "match_tflops_last_frame": match_flops / (match_ms[-1] / 1e3) / 1e12 if n_prev else None,
            "attn_unmerged_history_ms": full_ms, "attn_merged_history_ms": merged_ms,
            "attn_speedup": full_ms / merged_ms, "steps": args.steps, "warmup": args.warmup}


# --------------------------------------------------------------------------------------------- CPU / reference
def blas_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = [i.get("num_threads") for i in info if i.get("user_api") == "blas"]
        return int(max(n)) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def host_inputs(wl, seed):
    """One layer's inputs on the host with the ispa_inputs recipe: [K timeline, V timeline, W, Q per
    chunk] (float32 holding the stored values)."""
    k_tl = inp._store(wl, inp.kv_timeline(wl, 0, "k", seed))
    v_tl = inp._store(wl, inp.kv_timeline(wl, 0, "v", seed))
    qs = [inp.attention_inputs(wl, 0, c, seed, timelines=(k_tl, v_tl))["q"] for c in range(len(wl.chunks))]
    return [k_tl, v_tl, inp.weight(wl, 0, seed)] + qs


def oracle_step_time(wl, host_in, seed, n_sample):
    """The oracle as it stands on a bounded sample of one step: for every warmup chunk the attention
    passes (C1 local, C2 full) and the statistics on n_sample / chunks query rows, then the absorb,
    eps and selection in full.  Returns the step time extrapolated to all query rows (seconds), the
    seconds actually spent, and the sample description."""
    from oracle import ispa_oracle as orc
    k_tl, v_tl, W, *qs = host_in
    C = len(wl.chunks)
    per_chunk = max(1, n_sample // C)
    total, spent = 0.0, 0.0
    Al, Af, scale = [], [], []
    for c in range(C):
        hist, cur = wl.chunks[c]
        seg = lambda t, fr: (t[list(fr)].reshape(-1, wl.n_heads, wl.head_dim) if fr
                             else np.zeros((0, wl.n_heads, wl.head_dim), np.float32))
        n_q = wl.n_q(c)
        rows = inp.sample_rows(n_q, per_chunk, seed=seed, salt=777 + c)
        t0 = time.perf_counter()
        o = orc.dual_stream(qs[c], k_tl[0, :wl.n_sink], v_tl[0, :wl.n_sink], seg(k_tl, cur), seg(v_tl, cur),
                            seg(k_tl, hist), seg(v_tl, hist), rows=rows, with_hist=False)
        Al.append(orc.stack_heads(o["O_loc"]))
        Af.append(orc.stack_heads(o["O_full"]))
        dt = time.perf_counter() - t0
        spent += dt
        total += dt * n_q / len(rows)
        scale.append(n_q / len(rows))
    t0 = time.perf_counter()
    # statistics of the sampled rows, each chunk's rows weighted up to the chunk's row count
    w = np.concatenate([np.full(a.shape[0], math.sqrt(s)) for a, s in zip(Al, scale)])[:, None]
    G, R, S = orc.sufficient_stats(np.concatenate(Al) * w, np.concatenate(Af) * w)
    t1 = time.perf_counter()
    lam = orc.ridge_lambda(G, wl.lam_rel or 1e-2)
    dW = orc.absorb(G, R, W, lam)
    eps = orc.error_from_stats(G, R, S, W, dW)[0]
    orc.select_layers([eps], 1)
    orc.update_weight(W, dW)
    t2 = time.perf_counter()
    rows_all = wl.rows_per_layer
    rows_sampled = sum(min(per_chunk, wl.n_q(c)) for c in range(C))
    total += (t1 - t0) * rows_all / rows_sampled + (t2 - t1)
    spent += t2 - t0
    sample = (f"{per_chunk} query rows per warmup chunk ({C} chunks) x {wl.n_heads} heads through the local "
              f"and full softmax passes and the statistics (times scaled to all {rows_all} rows), plus one "
              f"full {wl.d}x{wl.d} absorb (LU solve), eps and selection")
    return total, spent, sample


def cpu_baseline(wl, host_in, seed, n_sample=1024):
    total, spent, sample = oracle_step_time(wl, host_in, seed, n_sample)
    return {"value": wl.rows_per_layer / total, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": sample, "cpu_seconds_spent": spent, "extrapolated_step_s": total}


def reference_arm(args):
    """--impl reference: the fp64 oracle as it stands, on the host cores, each step a bounded sample."""
    wl = inp.get_workload(args.workload)
    host_in = host_inputs(wl, args.seed)
    for _ in range(args.warmup):
        oracle_step_time(wl, host_in, args.seed, args.ref_rows)
    totals, spent, sample = [], 0.0, ""
    for _ in range(args.steps):
        t, s, sample = oracle_step_time(wl, host_in, args.seed, args.ref_rows)
        totals.append(t)
        spent += s
    ms = 1e3 * float(np.mean(totals))
    value = wl.rows_per_layer / (ms / 1e3)
    cores = blas_threads()
    return {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (the ispa_inputs recipe, drawn on the host)",
            "config": workload_config(wl), "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0, "cpu_seconds_spent": spent}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-rows", type=int, default=256)
    ap.add_argument("--ref-rows", type=int, default=128)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--overhead", action="store_true",
                    help="time plain attention against the dual-stream collection on one layer (prints its own line)")
    ap.add_argument("--stack", action="store_true",
                    help="multi-layer workloads: time the whole warmup of every layer instead of one layer")
    ap.add_argument("--infer", action="store_true",
                    help="with --stack: also time one inference chunk after T_warm (L-Layers vs all F-Layers)")
    ap.add_argument("--layers", type=int, default=0, help="with --stack: time only the first N layers")
    ap.add_argument("--overlap", action="store_true",
                    help="with --stack: statistics and absorbs on side streams, overlapping the attention")
    ap.add_argument("--tempcache", action="store_true",
                    help="time FAST-AR TempCache merging of the T_warm history and attention over it")
    ap.add_argument("--tc-threshold", type=float, default=0.9)
    ap.add_argument("--history-sweep", action="store_true",
                    help="dual-stream attention over 3..120 history frames: TFLOP/s and HBM GB/s")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(reference_arm(args)), flush=True)
        return
    if args.overhead:
        if rank == 0:
            print(json.dumps(overhead_arm(args)), flush=True)
        return
    if args.stack:
        if rank == 0:
            print(json.dumps(warmup_arm(args)), flush=True)
        return
    if args.tempcache:
        if rank == 0:
            print(json.dumps(tempcache_arm(args)), flush=True)
        return
    if args.history_sweep:
        if rank == 0:
            print(json.dumps(history_sweep_arm(args)), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = gpu_arm(args, rank, world, local_rank)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
