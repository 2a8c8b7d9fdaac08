"""The benchmark's reference arm (the oracle on the host cores) produces the contract's JSON line."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "1", "--warmup", "3", "--ref-rows", "8"], capture_output=True, text=True,
                       timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_time_interleaved_rotates_and_times_every_call():
    """The overhead mode's timing loop: each function warmed up, then every round runs all of them
    once, the starting function moving one place per round; each timed call is bracketed by its own
    events and preceded by an L2 flush.  A fake event clock stands in for CUDA events."""
    sys.path.insert(0, ROOT)
    import bench

    log = []

    class Clock:
        t = 0.0

    class Event:
        def __init__(self, enable_timing=False):
            assert enable_timing
            self.t = None

        def record(self):
            self.t = Clock.t

        def elapsed_time(self, other):
            return other.t - self.t

    class FakeCuda:
        @staticmethod
        def synchronize():
            log.append("sync")

    FakeCuda.Event = Event

    class FakeTorch:
        cuda = FakeCuda

    class Flush:
        def fill_(self, v):
            log.append("flush")

    def make(name, cost):
        def fn():
            log.append(name)
            Clock.t += cost
        return fn

    fns = [("a", make("a", 1.0)), ("b", make("b", 2.0)), ("c", make("c", 3.0))]
    ms = bench.time_interleaved(fns, steps=4, warmup=2, flush=Flush(), torch=FakeTorch)
    assert ms == {"a": [1.0] * 4, "b": [2.0] * 4, "c": [3.0] * 4}
    calls = [x for x in log if x not in ("sync", "flush")]
    assert calls[:6] == ["a", "a", "b", "b", "c", "c"]  # warm-up, each function in turn
    rounds = [calls[6 + 3 * i: 9 + 3 * i] for i in range(4)]
    assert rounds == [["a", "b", "c"], ["b", "c", "a"], ["c", "a", "b"], ["a", "b", "c"]]
    # every timed call: flush, call, synchronize
    timed = log[6:]
    assert len(timed) == 12 * 3 and all(timed[3 * i] == "flush" and timed[3 * i + 2] == "sync" for i in range(12))


def test_summarize_clocks_reports_load_median_and_active_reasons():
    """The bench line's clock record: median SM clock over the samples under load, the maximum clock,
    the throttle reasons seen active at least once, and malformed samples skipped."""
    sys.path.insert(0, ROOT)
    import bench

    na = "Not Active"
    lines = [
        f"0, 345, 1965, 110.5, 0x0, {na}, {na}, {na}, {na}",          # idle sample, excluded from the median
        f"0, 1965, 1965, 690.0, 0x0, {na}, {na}, {na}, {na}",
        f"0, 1890, 1965, 998.0, 0x4, {na}, {na}, {na}, Active",       # power cap
        f"0, 1950, 1965, 870.0, 0x0, {na}, {na}, {na}, {na}",
        "0, [N/A], 1965, [N/A], 0x0, Not Active, Not Active, Not Active, Not Active",  # malformed: skipped
        "garbage",
    ]
    c = bench.summarize_clocks(lines)
    assert c["sm_mhz"] == 1950.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"] and c["samples"] == 4
    assert c["power_w_median"] == (690.0 + 870.0) / 2
    hot = bench.summarize_clocks([f"0, 1500, 1965, 700, 0x40, {na}, Active, {na}, {na}"])
    assert hot["reasons"] == ["hw_thermal_slowdown"]
    assert bench.summarize_clocks([])["sm_mhz"] is None


def test_attention_traffic_capture_matches_the_committed_kernel():
    """The bench line's roofline traffic comes from the committed ncu capture only while the attention
    kernel's source is the one the counters were taken on; other workloads report none."""
    sys.path.insert(0, ROOT)
    import bench

    for wl in ("l14b", "l1_3b"):
        t = bench.attn_traffic(wl)
        cap = json.load(open(os.path.join(ROOT, "profiles", f"attn_tc_{wl}.json")))
        assert t is not None and t == cap["bytes_per_launch"], wl
        assert cap["dram_bytes_read"] + cap["dram_bytes_write"] == t
    assert bench.attn_traffic("tiny") is None
