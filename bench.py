"""Benchmark of the ISPA hot path on B200 (one JSON line on stdout from rank 0).

One step = one pass of the whole hot path over one batch of synthetic input, on the 1.3B-like layer
(d = 1536, 12 heads x 128, 4680 queries of the current chunk, 1560 sink + 4680 local + 14040 history
keys):
  1. decomposable dual-stream attention (A_loc, A_full, lse_loc, lse_hist, D = A_full - A_loc),
  2. warmup statistics G, R, S from A_loc and D,
  3. closed-form ridge absorb dW = (G + lam I)^-1 R W with lam = 1e-2 tr(G)/d, eps and eps_rel,
  4. layer selection (host) and W_new = W + dW.
value = query tokens per second of the whole step (all ranks).  Multi-GPU runs are replicas: each
rank processes its own independent layer, no collective on the data path (weak scaling).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]
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


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def workload_config(wl):
    return {"workload": f"{wl.name}: {wl.description}", "n_q": wl.n_q(0),
            "n_kv": [wl.n_sink, wl.n_local(0), wl.n_hist(0)], "d": wl.d, "heads": wl.n_heads,
            "head_dim": wl.head_dim, "lam_rel": wl.lam_rel or 1e-2,
            "l2": "flushed between timed steps (256 MiB write, outside the timed events)",
            "parallelism": "replicas (one independent layer per rank)"}


def attn_flops(wl):
    nk = wl.n_sink + wl.n_local(0) + wl.n_hist(0)
    return 4.0 * wl.n_q(0) * nk * wl.d


def stats_flops(wl):
    return 6.0 * wl.n_q(0) * wl.d * wl.d  # G, R, S as three full d x d Gram products


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
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        under_load = [m for m in mhz if m > 500] or mhz
        return {"sm_mhz": float(np.median(under_load)) if under_load else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(mhz)}


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


# --------------------------------------------------------------------------------------------- GPU arm
class Step:
    """Device buffers and the launch sequence of one hot-path step."""

    def __init__(self, wl, layer, seed, torch, ispa):
        self.torch, self.ispa, self.wl = torch, ispa, wl
        dev = "cuda"
        bf = torch.bfloat16
        x = inp.attention_inputs(wl, layer, 0, seed)
        self.host = {k: torch.from_numpy(v).to(bf).pin_memory() for k, v in x.items()}
        self.host["W"] = torch.from_numpy(inp.weight(wl, layer, seed)).to(bf).pin_memory()
        self.dev = {k: v.to(dev) for k, v in self.host.items()}
        n_q, d, H = wl.n_q(0), wl.d, wl.n_heads
        self.o_loc = torch.empty((n_q, d), dtype=bf, device=dev)
        self.o_full = torch.empty_like(self.o_loc)
        self.dd = torch.empty_like(self.o_loc)
        self.lse_loc = torch.empty((H, n_q), dtype=torch.float32, device=dev)
        self.lse_hist = torch.empty_like(self.lse_loc)
        self.GRS = [torch.empty((d, d), dtype=torch.float32, device=dev) for _ in range(3)]
        self.dW = torch.empty((d, d), dtype=torch.float32, device=dev)
        self.eps = torch.empty((4,), dtype=torch.float64, device=dev)
        self.w_new = torch.empty_like(self.dev["W"])
        self.ws = torch.empty((ispa.absorb_workspace_size(d),), dtype=torch.uint8, device=dev)
        self.eps_host = torch.empty((4,), dtype=torch.float64).pin_memory()
        self.dW_host = torch.empty((d, d), dtype=torch.float32).pin_memory()
        self.h2d_bytes = sum(v.numel() * v.element_size() for v in self.host.values())
        self.d2h_bytes = self.eps_host.numel() * 8 + self.dW_host.numel() * 4
        self.lam_rel = wl.lam_rel or 1e-2

    def run(self, ev=None, stream=None):
        """Launch one step on the current stream; `ev` (5 events) brackets the phases."""
        t, ispa = self.dev, self.ispa
        if ev:
            ev[0].record()
        ispa.dual_stream_attn(t["q"], t["k_sink"], t["v_sink"], t["k_loc"], t["v_loc"], t["k_hist"], t["v_hist"],
                              o_loc=self.o_loc, o_full=self.o_full, lse_loc=self.lse_loc, lse_hist=self.lse_hist,
                              d_out=self.dd)
        if ev:
            ev[1].record()
        ispa.accum_stats(self.o_loc, self.dd, *self.GRS, zero=True)
        if ev:
            ev[2].record()
        ispa.absorb(*self.GRS, t["W"], self.lam_rel, lam_rel=True, dW=self.dW, eps=self.eps, w_new=self.w_new,
                    write_wnew=True, ws=self.ws)
        if ev:
            ev[3].record()

    def finish_host(self):
        """Host side of the step: the selection over this rank's layer(s) from the eps read back."""
        e = float(self.eps_host[0])
        idx, mask, st = self.ispa.select_layers([e], 1)
        return idx

    def run_e2e(self):
        """Same step through the public API from pinned host memory: H2D inputs, step, D2H result."""
        for k, v in self.host.items():
            self.dev[k].copy_(v, non_blocking=True)
        self.run()
        self.eps_host.copy_(self.eps, non_blocking=True)
        self.dW_host.copy_(self.dW, non_blocking=True)


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
    step = Step(wl, layer=rank, seed=args.seed, torch=torch, ispa=ispa)
    flush = torch.empty((L2_FLUSH_BYTES // 4,), dtype=torch.float32, device="cuda")
    K, W = args.steps, args.warmup

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(W):
        flush.fill_(1.0)
        step.run()
    torch.cuda.synchronize()
    if ispa.get_device_status() != 0:
        raise RuntimeError("device status after warm-up: " + ispa.status_string(ispa.get_device_status()))

    # ---- timed region: K steps, each bracketed by events; L2 flushed between steps, outside the events
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
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
    step_ms = [e[0].elapsed_time(e[3]) for e in evs]
    attn_ms = [e[0].elapsed_time(e[1]) for e in evs]
    stats_ms = [e[1].elapsed_time(e[2]) for e in evs]
    absorb_ms = [e[2].elapsed_time(e[3]) for e in evs]
    host_sel = step.finish_host()

    # ---- end to end through the public API with host buffers (H2D inputs, D2H dW and eps)
    for _ in range(max(1, W)):
        step.run_e2e()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(K):
        step.run_e2e()
    e1.record()
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1) / K
    step.finish_host()

    total_ms = float(sum(step_ms))
    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], world, "cuda")
    if rank != 0:
        return None
    peaks = load_peaks()
    n_q = wl.n_q(0)
    ms_per_step = total_ms / K
    value = aggregate_value(world, n_q, K, total_ms)
    attn_avg = float(np.mean(attn_ms))
    af = attn_flops(wl)
    achieved = af / (attn_avg / 1e3) / 1e12
    traffic = attn_traffic(wl.name)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic: seeded AR(1) K/V across latent frames, Gaussian Q and W, "
                                 "shapes of a Wan/LongLive-1.3B-like layer",
        "config": workload_config(wl),
        "roofline": {"bound": "tensor", "kernel": "attn_tc_kernel<128>", "achieved": achieved,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                     "peak_source": f"{peaks['source']} bf16 matmul burst (MEASURED_PEAKS.json)",
                     "algorithmic_flops_per_launch": af, "traffic": traffic},
        "attn_ms": attn_avg, "attn_tflops": achieved, "attn_frac_bf16_peak": achieved / peaks["bf16_tflops"],
        "stats_ms": float(np.mean(stats_ms)),
        "stats_tflops": stats_flops(wl) / (float(np.mean(stats_ms)) / 1e3) / 1e12,
        "absorb_ms_per_layer": float(np.mean(absorb_ms)),
        "e2e": {"value": world * n_q / (e2e_ms / 1e3), "unit": UNIT, "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": step.h2d_bytes, "d2h_bytes_per_step": step.d2h_bytes},
        "gpu_launches": int(launches),
        "clocks": clocks,
        "selected": [int(i) for i in host_sel],
    }
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(wl, args.seed, n_sample=args.cpu_rows)
    return line


# --------------------------------------------------------------------------------------------- multi-layer warmups
def gpu_inputs(wl, layer, seed, torch):
    """The input recipe of ispa_inputs drawn on the GPU (seeded torch generator) for the multi-layer
    timing runs: AR(1) K/V timelines across latent frames, Gaussian Q per chunk, W ~ N(0, 1/d); bf16."""
    g = torch.Generator(device="cuda")
    g.manual_seed((seed * 1000003 + layer) & 0x7FFFFFFF)
    shape = (wl.n_frames, wl.frame_tokens, wl.n_heads, wl.head_dim)
    tl = []
    for _ in range(2):
        x = torch.empty(shape, dtype=torch.float32, device="cuda")
        x[0].normal_(generator=g)
        a, b = wl.rho, math.sqrt(1.0 - wl.rho * wl.rho)
        for f in range(1, wl.n_frames):
            x[f].normal_(generator=g).mul_(b).add_(x[f - 1], alpha=a)
        tl.append(x.to(torch.bfloat16))
        del x
    s = inp.logit_scale(wl, layer, seed)
    qs = [(torch.randn((wl.n_q(c), wl.n_heads, wl.head_dim), generator=g, device="cuda") * s).to(torch.bfloat16)
          for c in range(len(wl.chunks))]
    W = (torch.randn((wl.d, wl.d), generator=g, device="cuda") / math.sqrt(wl.d)).to(torch.bfloat16)
    return tl, qs, W


def segments(wl, tl, c):
    """Sink, local and history K/V segments of chunk c as views into a layer's timeline."""
    hist, cur = wl.chunks[c]
    F, P = wl.frame_tokens, wl.n_heads
    def frames(t, fr):
        if not fr:
            return t[0, :0]
        return t[fr[0]:fr[-1] + 1].reshape(-1, wl.n_heads, wl.head_dim)
    return [(t[0, :wl.n_sink], frames(t, cur), frames(t, hist)) for t in tl]


def overhead_arm(args):
    """Cost of collecting both streams (the pages call it negligible): on one layer of the workload,
    plain single-branch attention over every key (sink and history in one segment, so the kernel
    keeps one softmax state) against the dual-stream pass, the dual-stream pass with D, and the
    dual-stream pass with D plus the Gram statistics.  CUDA events, L2 flushed between repetitions."""
    import torch
    import kv_cache_compression_tma_b200 as ispa
    wl = inp.get_workload(args.workload)
    step = Step(wl, layer=0, seed=args.seed, torch=torch, ispa=ispa)
    t = step.dev
    one = torch.cat([t["k_sink"], t["k_hist"]], 0), torch.cat([t["v_sink"], t["v_hist"]], 0)
    empty_k, empty_v = t["k_loc"][:0], t["v_loc"][:0]
    flush = torch.empty((L2_FLUSH_BYTES // 4,), dtype=torch.float32, device="cuda")
    out = dict(o_loc=step.o_loc, o_full=step.o_full, lse_loc=step.lse_loc, lse_hist=step.lse_hist)

    def plain():
        ispa.dual_stream_attn(t["q"], one[0], one[1], t["k_loc"], t["v_loc"], empty_k, empty_v, want_delta=False,
                              **out)

    def dual():
        ispa.dual_stream_attn(t["q"], t["k_sink"], t["v_sink"], t["k_loc"], t["v_loc"], t["k_hist"], t["v_hist"],
                              want_delta=False, **out)

    def dual_d():
        ispa.dual_stream_attn(t["q"], t["k_sink"], t["v_sink"], t["k_loc"], t["v_loc"], t["k_hist"], t["v_hist"],
                              d_out=step.dd, **out)

    def dual_d_stats():
        dual_d()
        ispa.accum_stats(step.o_loc, step.dd, *step.GRS, zero=True)

    res = {}
    for name, fn in (("plain_attention", plain), ("dual_stream", dual), ("dual_stream_with_d", dual_d),
                     ("dual_stream_with_d_and_stats", dual_d_stats)):
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
        res[name + "_ms"] = float(np.mean(ms))
    if ispa.get_device_status() != 0:
        raise RuntimeError("device status after the overhead runs")
    base = res["plain_attention_ms"]
    for name in ("dual_stream", "dual_stream_with_d", "dual_stream_with_d_and_stats"):
        res[name + "_overhead"] = res[name + "_ms"] / base - 1.0
    return {"mode": "collection_overhead", "workload": wl.name, "steps": args.steps, "warmup": args.warmup, **res}


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
    w_new = [torch.empty_like(layers[l][2]) for l in range(L)]

    def run(ev=None):
        for l in range(L):
            tl, qs, W = layers[l]
            for c in range(len(wl.chunks)):
                (ks, kl, kh), (vs, vl, vh) = segments(wl, tl, c)
                n = wl.n_q(c)
                ispa.dual_stream_attn(qs[c], ks, vs, kl, vl, kh, vh, o_loc=o_loc[:n], o_full=o_full[:n],
                                      lse_loc=lse_l[:, :n], lse_hist=lse_h[:, :n], d_out=dd[:n])
                ispa.accum_stats(o_loc[:n], dd[:n], *stats[l], zero=(c == 0))
        if ev:
            ev[1].record()
        for l in range(L):
            ispa.absorb(*stats[l], layers[l][2], wl.lam_rel, lam_rel=True, dW=dW, eps=eps[l], w_new=w_new[l],
                        write_wnew=True, ws=ws)
        if ev:
            ev[2].record()
        e = eps[:, 0].cpu().numpy()
        return ispa.select_layers(e, min(wl.k_select or L, max(1, L // 2)) if L < wl.n_layers else (wl.k_select or max(1, L // 2)))

    for _ in range(max(1, args.warmup)):
        run()
    torch.cuda.synchronize()
    times = []
    for _ in range(args.steps):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record()
        idx, mask, st = run(ev)
        torch.cuda.synchronize()
        times.append((ev[0].elapsed_time(ev[1]), ev[1].elapsed_time(ev[2]), ev[0].elapsed_time(ev[2])))
    if ispa.get_device_status() != 0:
        raise RuntimeError("device status after the warmup runs")
    infer = infer_arm(args, wl, L, layers, w_new, idx, torch) if args.infer else None
    t_attn = float(np.mean([t[0] for t in times]))
    t_abs = float(np.mean([t[1] for t in times]))
    t_all = float(np.mean([t[2] for t in times]))
    rows = sum(wl.n_q(c) for c in range(len(wl.chunks)))
    flops = sum(4.0 * wl.n_q(c) * (wl.n_sink + wl.n_local(c) + wl.n_hist(c)) * d for c in range(len(wl.chunks)))
    peaks = load_peaks()
    cfg = workload_config(wl)
    cfg.update({"layers_timed": L, "chunks": len(wl.chunks), "k_select": wl.k_select})
    return {"metric": METRIC, "value": L * rows / (t_all / 1e3), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t_all, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic, drawn on the GPU with the ispa_inputs recipe",
            "config": cfg, "attn_plus_stats_ms": t_attn,
            "attn_stats_tflops": L * flops / (t_attn / 1e3) / 1e12, "absorb_ms_total": t_abs,
            "absorb_ms_per_layer": t_abs / L, "selected": [int(i) for i in idx],
            "note": "attention figures include the statistics GEMMs; L2 not flushed between layers",
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
            tl, qs, W = layers[l]
            (ks, kl, kh), (vs, vl, vh) = segments(wl, tl, c)
            is_l = mixed and l in sel
            ll.layer_forward(qs[c], ks, vs, kl, vl, kh, vh, w_new[l] if is_l else W, llayer=is_l, work=work, out=y)

    res = {}
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
    W0 = layers[0][2]
    for _ in range(3):
        ispa.project(a, W0, out=y)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 50
    e0.record()
    for _ in range(reps):
        ispa.project(a, W0, out=y)
    e1.record()
    torch.cuda.synchronize()
    proj_ms = e0.elapsed_time(e1) / reps
    peak = load_peaks()["bf16_tflops"]
    proj_tflops = 2.0 * n * wl.d * wl.d / (proj_ms / 1e3) / 1e12
    res.update({"project_ms": proj_ms, "project_tflops": proj_tflops, "project_frac_bf16_peak": proj_tflops / peak})
    if ispa.get_device_status() != 0:
        raise RuntimeError("device status after the inference steps")
    res.update(ll.kv_savings(sel, L, ll.kv_bytes(wl.n_sink, wl.n_local(c), wl.n_hist(c), wl.n_heads, wl.head_dim, 2)))
    res["l_layers"] = len(sel)
    res["query_tok_per_s_mixed"] = L * n / (res["ms_mixed"] / 1e3)
    res["query_tok_per_s_all_full"] = L * n / (res["ms_all_full"] / 1e3)
    return res


# --------------------------------------------------------------------------------------------- CPU / reference
def blas_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = [i.get("num_threads") for i in info if i.get("user_api") == "blas"]
        return int(max(n)) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_step_time(wl, seed, n_sample, x=None, W=None):
    """The oracle as it stands on a bounded sample of one step: the attention passes (C1 local, C2 full)
    and the statistics on `n_sample` query rows, the absorb, eps and selection in full.  Returns the
    step time extrapolated to all query rows (seconds) and the sample description."""
    from oracle import ispa_oracle as orc
    if x is None:
        x = inp.attention_inputs(wl, 0, 0, seed)
    if W is None:
        W = inp.weight(wl, 0, seed)
    n_q = wl.n_q(0)
    rows = inp.sample_rows(n_q, n_sample, seed=seed, salt=777)
    t0 = time.perf_counter()
    o = orc.dual_stream(x["q"], x["k_sink"], x["v_sink"], x["k_loc"], x["v_loc"], x["k_hist"], x["v_hist"],
                        rows=rows, with_hist=False)
    t1 = time.perf_counter()
    A_loc, A_full = orc.stack_heads(o["O_loc"]), orc.stack_heads(o["O_full"])
    G, R, S = orc.sufficient_stats(A_loc, A_full)
    t2 = time.perf_counter()
    # the absorb needs statistics of full rank: scale the sample's Gram to the chunk's row count and
    # regularise as the step does (the solve's cost does not depend on the values)
    scale = n_q / len(rows)
    G, R, S = G * scale, R * scale, S * scale
    lam = orc.ridge_lambda(G, wl.lam_rel or 1e-2)
    dW = orc.absorb(G, R, W, lam)
    eps = orc.error_from_stats(G, R, S, W, dW)[0]
    orc.select_layers([eps], 1)
    orc.update_weight(W, dW)
    t3 = time.perf_counter()
    frac = n_q / len(rows)
    total = (t1 - t0) * frac + (t2 - t1) * frac + (t3 - t2)
    sample = (f"{len(rows)} of {n_q} query rows x {wl.n_heads} heads through the local and full softmax "
              f"passes and the statistics (times x {frac:.3g}), plus one full {wl.d}x{wl.d} absorb "
              f"(LU solve), eps and selection")
    return total, t3 - t0, sample


def cpu_baseline(wl, seed, n_sample=1024):
    total, spent, sample = oracle_step_time(wl, seed, n_sample)
    return {"value": wl.n_q(0) / total, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": sample, "cpu_seconds_spent": spent, "extrapolated_step_s": total}


def reference_arm(args):
    """--impl reference: the fp64 oracle as it stands, on the host cores, each step a bounded sample."""
    wl = inp.get_workload(args.workload)
    x = inp.attention_inputs(wl, 0, 0, args.seed)
    W = inp.weight(wl, 0, args.seed)
    n_sample = args.ref_rows
    for _ in range(args.warmup):
        oracle_step_time(wl, args.seed, n_sample, x, W)
    totals, spent, sample = [], 0.0, ""
    for _ in range(args.steps):
        t, s, sample = oracle_step_time(wl, args.seed, n_sample, x, W)
        totals.append(t)
        spent += s
    ms = 1e3 * float(np.mean(totals))
    value = wl.n_q(0) / (ms / 1e3)
    cores = blas_threads()
    return {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (same seeded inputs as the GPU arm)",
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
    ap.add_argument("--workload", default="l1_3b")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-rows", type=int, default=1024)
    ap.add_argument("--ref-rows", type=int, default=512)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--overhead", action="store_true",
                    help="time plain attention against the dual-stream collection on one layer (prints its own line)")
    ap.add_argument("--infer", action="store_true",
                    help="multi-layer workloads: also time one inference chunk after T_warm (L-Layers vs all F-Layers)")
    ap.add_argument("--layers", type=int, default=0, help="multi-layer workloads: time only the first N layers")
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
    wl = inp.get_workload(args.workload)
    if args.overhead:
        if rank == 0:
            print(json.dumps(overhead_arm(args)), flush=True)
        return
    if wl.n_layers > 1 or len(wl.chunks) > 1:
        if rank == 0:
            print(json.dumps(warmup_arm(args)), flush=True)
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
