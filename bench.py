"""Benchmark of the fused attention forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the decode sweep (B=1, Hq=64, Hkv in {4, 8}, L=1,
S in {256 ... 32768}, Dqk=192 / Dv=128, bf16, causal): twelve attention calls
through the C ABI, each a split-KV pass plus a log-sum-exp combine chosen by
the router.  The headline is KV HBM GB/s (KV bytes the calls must read /
device time).  L2 is flushed (a 2x L2-sized buffer is written) before every
call, outside the timed kernels.  The same JSON line also carries the
prefill configurations (TFLOP/s against the tensor peak), the verify sweep
and the encoder shapes as secondary objects, the roofline of the dominant
kernel, an end-to-end number through the public API with host buffers, and
the fp64 CPU oracle timed on a bounded sample.

With N > 1 (torchrun, one process per GPU) every rank runs the same sweep
on its own GPU: the (batch, KV head) units are independent, so there is no
collective on the data path ("scaling": "weak"); timing is the max over
ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from scaled_dot_product_13_b200 import inputs as I  # noqa: E402
from scaled_dot_product_13_b200.accounting import flops, io_bytes, kv_bytes  # noqa: E402

METRIC = "prefill TFLOP/s & decode KV HBM GB/s on 1 B200, % of roofline; µs per SDPA call"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def ncu_traffic(kernel_file: str, tag: str):
    """Per-launch DRAM bytes from a committed ncu summary, only while the
    kernel source it was taken on is unchanged (sha256 recorded beside it)."""
    prof = os.path.join(ROOT, "profiles", "traffic.md")
    try:
        text = open(prof).read()
    except OSError:
        return None
    src = open(os.path.join(ROOT, "scaled_dot_product_13_b200", "csrc", kernel_file), "rb").read()
    sha = hashlib.sha256(src).hexdigest()[:16]
    for m in re.finditer(r"^traffic (\S+) (\S+) bytes_per_launch=(\d+) source_sha256=(\w+)",
                         text, re.M):
        if m.group(1) == tag and m.group(2) == kernel_file and m.group(4) == sha:
            return int(m.group(3))
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


class Case:
    """One attention problem resident on the device, ready to call."""

    def __init__(self, sdpa, p: I.Problem, device):
        self.p = p
        q, k, v = I.make_qkv(p)
        self.q, self.k, self.v = q.to(device), k.to(device), v.to(device)
        self.out = torch.empty(p.B, p.Hq, p.L, p.Dv, dtype=p.torch_dtype, device=device)
        self.info = sdpa.plan(p.B, p.Hq, p.Hkv, p.L, p.S, p.Dqk, p.Dv, p.causal, p.window, p.dtype)
        nb = self.info["workspace_bytes"]
        self.ws = torch.empty(max(nb, 4) // 4, dtype=torch.float32, device=device) if nb else None
        self.kv_bytes = kv_bytes(p)
        self.flops = flops(p)
        self.io_bytes = io_bytes(p)

    def call(self, sdpa):
        sdpa.forward_ws(self.q, self.k, self.v, self.ws, scale=self.p.sm_scale,
                        causal=self.p.causal, window_size=self.p.window, out=self.out)


def flush_l2(buf):
    """Evict L2: write a buffer larger than L2, then read it back so that the
    lines left in L2 are clean (the next kernel pays no write-back)."""
    buf.zero_()
    return buf.sum()


def max_over_ranks(x: float, dist, device) -> float:
    """Max of a per-rank float over all ranks (identity without a group)."""
    if dist is None:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world: int, bytes_per_rank_step: float, steps: int, max_total_ms: float) -> float:
    """Whole-job throughput: every rank's bytes over the slowest rank's time."""
    return world * bytes_per_rank_step * steps / (max_total_ms * 1e-3) / 1e9


class HostCase:
    """A problem's seeded inputs on the host (for the CPU oracle)."""

    def __init__(self, p: I.Problem):
        self.p = p
        self.q, self.k, self.v = I.make_qkv(p)
        self.kv_bytes = kv_bytes(p)


def time_cases(sdpa, cases, steps, warmup, flush, sync_all, graphs=True):
    """Per call: flush L2 (untimed), then run the call with CUDA events
    recorded by the library on its launch stream.

    Two runners per call, replayed in turn.  The timed one records an event before
    the main kernel and one after the call's last launch (the combine, when
    split): call time = the device time of the library's work.  Nothing sits
    between the split pass and the combine there, so the combine keeps its
    programmatic (early) launch.  The second runner adds an event right after
    the main kernel, which serialises the combine behind it; it only gives the
    main kernel's own time for the roofline.  With ``graphs`` each runner is
    captured once into a CUDA graph and replayed, so the device timeline
    carries no host enqueue gaps.  Returns per-case lists (ms): call, main,
    outer (the timed replay including graph-launch edges)."""
    call_ms = [[] for _ in cases]
    main_ms = [[] for _ in cases]
    outer_ms = [[] for _ in cases]
    stream = torch.cuda.current_stream()
    hooks = []
    for c in cases:
        evs = tuple(torch.cuda.Event(enable_timing=True) for _ in range(5))
        for e in evs:
            e.record(stream)  # creates the CUDA handles; the library re-records them
        c.call(sdpa)  # first call outside any capture (kernel attributes, TMA encode path)
        hooks.append(evs)
    torch.cuda.synchronize()

    def runner(c, a, b, d):
        if graphs:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                sdpa.time_next_call(a, b, d)
                c.call(sdpa)
            return g.replay

        def eager():
            sdpa.time_next_call(a, b, d)
            c.call(sdpa)
        return eager

    timed = [runner(c, h[0], None, h[1]) for c, h in zip(cases, hooks)]
    probes = [runner(c, h[2], h[3], h[4]) for c, h in zip(cases, hooks)]
    torch.cuda.synchronize()
    # One call at a time: its warm-up replays, then its timed ones.  Replays of
    # different calls interleaved would make a call pay for the SMs' switch
    # between shared-memory configurations of unlike kernels (one-tile
    # tcgen05 after split-KV, say), which a call repeated in a loop does not.
    for i, (run, probe) in enumerate(zip(timed, probes)):
        h = hooks[i]
        for it in range(warmup + steps):
            flush_l2(flush)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            run()
            e1.record(stream)
            flush_l2(flush)
            probe()
            if it == warmup - 1:
                sync_all()
            if it >= warmup:
                torch.cuda.synchronize()
                call_ms[i].append(h[0].elapsed_time(h[1]))
                main_ms[i].append(h[2].elapsed_time(h[3]))
                outer_ms[i].append(e0.elapsed_time(e1))
    return call_ms, main_ms, outer_ms


def time_steps(sdpa, cases, steps, warmup, flush, sync_all, graphs=True):
    """The headline step: every call of the sweep back to back on one stream
    (captured once into a CUDA graph and replayed), L2 flushed before each
    step outside the timed region.  The step's inputs are larger than L2 and
    each call's inputs were last read a whole step earlier, so every call
    reads its KV from HBM.  The K timed steps are bracketed by a barrier and a
    synchronize on both sides; returns the per-step device times (ms)."""
    stream = torch.cuda.current_stream()

    def body():
        for c in cases:
            c.call(sdpa)

    run = body
    if graphs:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            body()
        run = g.replay
    torch.cuda.synchronize()
    for _ in range(warmup):
        flush_l2(flush)
        run()
    sync_all()
    evs = []
    for _ in range(steps):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run()
        e1.record(stream)
        evs.append((e0, e1))
    sync_all()
    return [e0.elapsed_time(e1) for e0, e1 in evs]


def time_e2e(sdpa, cases, steps, warmup, device):
    """Public API with host buffers: pinned host -> device copy of q, k, v,
    the call, device -> host copy of out; all inside the timed region."""
    hosts = []
    for c in cases:
        hosts.append(tuple(t.cpu().pin_memory() for t in (c.q, c.k, c.v)) +
                     (torch.empty(c.out.shape, dtype=c.out.dtype).pin_memory(),))
    stream = torch.cuda.current_stream()
    tot = []
    h2d = d2h = 0
    for it in range(warmup + steps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for c, (hq, hk, hv, ho) in zip(cases, hosts):
            qd = hq.to(device, non_blocking=True)
            kd = hk.to(device, non_blocking=True)
            vd = hv.to(device, non_blocking=True)
            out = sdpa.forward(qd, kd, vd, scale=c.p.sm_scale, causal=c.p.causal,
                               window_size=c.p.window)
            ho.copy_(out, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        if it >= warmup:
            tot.append(e0.elapsed_time(e1))
    for c in cases:
        h2d += sum(t.numel() * t.element_size() for t in (c.q, c.k, c.v))
        d2h += c.out.numel() * c.out.element_size()
    return tot, h2d, d2h


def oracle_sample(cases, budget_s=12.0):
    """The fp64 CPU oracle as it stands, on a bounded sample of the decode
    sweep: every call of the sweep, repeated while the budget lasts (one
    full pass at least).  Returns (KV GB/s, seconds, cores, calls)."""
    from oracle import sdpa_oracle

    cores = os.cpu_count() or 1
    host = [(tuple(t.cpu() for t in (c.q, c.k, c.v)), c) for c in cases]
    t0 = time.perf_counter()
    nbytes, calls = 0.0, 0
    while True:
        for (q, k, v), c in host:
            sdpa_oracle(q, k, v, c.p.sm_scale, c.p.causal, c.p.window, nthreads=cores)
            nbytes += c.kv_bytes
            calls += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return nbytes / dt / 1e9, dt, cores, calls


def verify_checks(points):
    """Monotonicity and cliff checks of the verify sweep, per S.

    Monotone: t(L_next) >= 0.97 t(L) for consecutive L.  No cliff over
    L in [8, 64]: t(L_next) / t(L) <= max(1.25, L_next / L) (the pages' cliff
    was a 2.3x jump for 1.5x the rows).  Points are named verify_s<S>_l<L>."""
    by_s = {}
    for p in points:
        s_part, l_part = p["name"].split("_")[1:3]
        by_s.setdefault(int(s_part[1:]), []).append((int(l_part[1:]), p["us"]))
    out = {}
    for S, pts in sorted(by_s.items()):
        pts.sort()
        mono = all(b[1] >= 0.97 * a[1] for a, b in zip(pts, pts[1:]))
        ratios = [(a[0], b[0], b[1] / a[1]) for a, b in zip(pts, pts[1:]) if a[0] >= 8]
        cliff = [r for r in ratios if r[2] > max(1.25, r[1] / r[0])]
        worst = max(ratios, key=lambda r: r[2] / max(1.25, r[1] / r[0])) if ratios else None
        out[f"s{S}"] = {"monotone": mono, "no_cliff": not cliff,
                        "worst_step": None if worst is None else
                        {"from_L": worst[0], "to_L": worst[1], "ratio": round(worst[2], 3)}}
    return out


def time_stream(sdpa, c, flush, l2_bytes, reps=6, warmup=2, max_copies=32,
                max_bytes=4 << 30):
    """Back-to-back throughput of one call: n calls in a row on n copies of the
    inputs whose total exceeds 2x L2 (so every call reads its inputs from HBM),
    captured in one CUDA graph; events around each replay, L2 flushed before
    it.  Returns microseconds per call (mean over ``reps`` replays).  One call
    alone carries its launch edges; here they overlap the neighbouring calls,
    as in a model that runs attention layer after layer."""
    per = sum(t.numel() * t.element_size() for t in (c.q, c.k, c.v))
    n = max(1, min(max_copies, -(-2 * l2_bytes // per) + 1, max(1, max_bytes // per)))
    copies = [(c.q, c.k, c.v)] + [tuple(t.clone() for t in (c.q, c.k, c.v)) for _ in range(n - 1)]
    stream = torch.cuda.current_stream()

    def body():
        for q, k, v in copies:
            sdpa.forward_ws(q, k, v, c.ws, scale=c.p.sm_scale, causal=c.p.causal,
                            window_size=c.p.window, out=c.out)

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        body()
    torch.cuda.synchronize()
    ts = []
    for it in range(warmup + reps):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        if it >= warmup:
            ts.append(e0.elapsed_time(e1) * 1e3 / n)
    del g, copies
    return statistics.mean(ts), n


def time_alone(sdpa, c, flush, reps=20, warmup=3):
    """One call captured alone in a CUDA graph, replayed after an L2 flush,
    with events around the replay on the stream (no event inside the graph).
    Returns microseconds per call (mean over ``reps``)."""
    stream = torch.cuda.current_stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        sdpa.forward_ws(c.q, c.k, c.v, c.ws, scale=c.p.sm_scale, causal=c.p.causal,
                        window_size=c.p.window, out=c.out)
    torch.cuda.synchronize()
    ts = []
    for it in range(warmup + reps):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        if it >= warmup:
            ts.append(e0.elapsed_time(e1) * 1e3)
    del g
    return statistics.mean(ts)


def secondary(sdpa, probs, steps, warmup, flush, sync_all, device, peaks, kind, graphs=True,
              stream=False):
    """Time a list of problems (one call each per step); return a summary.
    With ``stream``, each problem is also timed back to back (``us_stream``)."""
    cases = [Case(sdpa, p, device) for p in probs]
    # Each timing pass goes over the list in order, heaviest call last, with a
    # pause after it: seconds of full tensor load lower the clock under the
    # power cap for a while, which would slow the next pass's first calls.
    # A call timed alone takes the median of its means over three such passes,
    # so that a drift of the clock during one pass does not land on one call
    # (calls of the same work, e.g. verify L = 12..32 on one 128-row tile,
    # otherwise differed by up to 3.5 %).
    alone = None
    if graphs:
        passes = 3
        reps = max(steps, 20) // passes + 1
        per = [[] for _ in cases]
        for _ in range(passes):
            for i, c in enumerate(cases):
                per[i].append(time_alone(sdpa, c, flush, reps=reps))
            time.sleep(1.0)
        alone = [statistics.median(x) for x in per]
    call_ms, main_ms, _ = time_cases(sdpa, cases, steps, warmup, flush, sync_all, graphs)
    time.sleep(1.0)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    pts = []
    for i, (c, cm, mm) in enumerate(zip(cases, call_ms, main_ms)):
        # the call timed alone: a graph holding only the call, replayed after
        # an L2 flush, events on the stream around the replay.  us_events is
        # the same call bracketed by events the library records inside the
        # graph, which carry several microseconds of their own (mean over the
        # timed steps: the device timer's coarse steps make a median jump
        # between neighbouring values)
        us = alone[i] if graphs else 1e3 * statistics.mean(cm)
        d = {"name": c.p.name, "us": round(us, 2),
             "us_events": round(1e3 * statistics.mean(cm), 2),
             "us_events_median": round(1e3 * statistics.median(cm), 2),
             "path": c.info["path"], "splits": c.info["splits"]}
        if kind == "tflops":
            tf = c.flops / (us * 1e-6) / 1e12
            d.update({"tflops": round(tf, 1),
                      "frac_tensor": round(tf / peaks["bf16_tflops"], 4)})
        d["kv_gbs"] = round(c.kv_bytes / (us * 1e-6) / 1e9, 1)
        d["frac_hbm"] = round(d["kv_gbs"] / peaks["hbm_gbs"], 4)
        # the call's own roofline: the slower of streaming its KV at the
        # measured copy bandwidth and its FLOPs at the measured tensor peak
        # (verify shapes sit near the ridge)
        floor_us = 1e6 * max(c.kv_bytes / (peaks["hbm_gbs"] * 1e9),
                             c.flops / (peaks["bf16_tflops"] * 1e12))
        d["roofline_us"] = round(floor_us, 2)
        d["frac_roofline"] = round(floor_us / us, 4)
        if stream:
            us_s, n = time_stream(sdpa, c, flush, l2)
            d["us_stream"] = round(us_s, 2)
            d["stream_copies"] = n
            d["frac_roofline_stream"] = round(floor_us / us_s, 4)
            if kind == "tflops":
                d["tflops_stream"] = round(c.flops / (us_s * 1e-6) / 1e12, 1)
        pts.append(d)
    del cases
    torch.cuda.empty_cache()
    return pts


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the prefill / verify / encoder objects")
    ap.add_argument("--only", default=None,
                    help="restrict the timed sweep to the named problem (profiling)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing")
    ap.add_argument("--eager", action="store_true",
                    help="time eager calls instead of replaying one CUDA graph per call")
    args = ap.parse_args()
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    probs = I.decode_problems()
    if args.only:
        probs = [p for p in probs + I.verify_problems() + I.window_problems() +
                 I.encoder_problems() + [I.tiny_problem()] + I.wide_problems()
                 if p.name == args.only]
        if not probs:
            raise SystemExit(f"unknown problem {args.only}")
    peaks, peak_src = load_peaks()
    workload = {"workload": "decode split-KV sweep: B=1, Hq=64, Hkv in {4,8}, L=1, "
                            "S in {256,1024,4096,8192,16384,32768}, Dqk=192, Dv=128, bf16, causal",
                "calls_per_step": len(probs),
                "l2": "flushed before every step (2x L2 buffer written, then read; the step's "
                      "474 MB of KV exceed L2) and before every call timed alone",
                "launch": "eager" if args.eager else "the step's calls captured in one CUDA graph, replayed",
                "timing": "step = events around the back-to-back calls of one step; per call "
                          "(points) = library events before the split pass and after the call's "
                          "last launch, each call replayed alone after an L2 flush, mean over the "
                          "timed steps; main-kernel time from probe replays with an event after "
                          "the split pass; prefill, verify, tiny and wide us = a graph of the call "
                          "alone replayed after an L2 flush, events around the replay (us_events: "
                          "library events inside the graph); us_stream = calls back to back on "
                          "rotating input copies totalling more than 2x L2, per call",
                "parallelism": f"replicas x{world} (independent KV-head units, no collective)"}

    if args.impl == "reference":
        if rank == 0:
            host_cases = [HostCase(p) for p in probs]
            for _ in range(args.warmup):
                oracle_sample(host_cases[:1], budget_s=0.0)
            vals, secs = [], 0.0
            cores = os.cpu_count() or 1
            for _ in range(args.steps):
                v_, dt, cores, _ = oracle_sample(host_cases, budget_s=0.0)
                vals.append(v_)
                secs += dt
            val = statistics.median(vals)
            line = {"impl": "reference", "metric": METRIC, "value": round(val, 4),
                    "unit": "GB/s (KV, decode)", "n_gpus": args.gpus, "steps": args.steps,
                    "warmup": args.warmup, "ms_per_step": round(1e3 * secs / args.steps, 3),
                    "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                    "dtype": "f64", "data": "synthetic N(0,1), seeded", "config": workload,
                    "cpu_baseline": {"kind": "oracle", "value": round(val, 4),
                                     "unit": "GB/s (KV, decode)", "cores": cores,
                                     "sample": "one full pass of the 12-call decode sweep per step"},
                    "e2e": {"value": round(val, 4), "unit": "GB/s (KV, decode)",
                            "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
            print(json.dumps(line), flush=True)
        # the oracle runs on the host: no device and no process group are
        # needed, and ranks other than 0 exit without work
        return

    dist = None
    if world > 1:
        import torch.distributed as dist  # noqa: F811
        import datetime

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)

    import scaled_dot_product_13_b200 as sdpa

    sdpa.load_library()
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20) // 4, dtype=torch.float32, device=device)

    def sync_all():
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
            torch.cuda.synchronize()

    cases = [Case(sdpa, p, device) for p in probs]
    sync_all()
    sampler = ClockSampler(device.index if device.index is not None else 0)
    # warm-up steps run inside time_cases; the sampler covers the timed steps
    sampler.start()
    step_ms = time_steps(sdpa, cases, args.steps, args.warmup, flush, sync_all,
                         graphs=not args.eager)
    call_ms, main_ms, outer_ms = time_cases(sdpa, cases, args.steps, args.warmup, flush,
                                            sync_all, graphs=not args.eager)
    sync_all()
    clocks = sampler.stop()
    sdpa.device_status(clear=False)

    # the sum of the calls timed one by one (each cold, each with its own
    # launch edges): a per-call view beside the step's back-to-back time
    calls_sum_ms = float(np.mean([sum(cm[s] for cm in call_ms) for s in range(args.steps)]))
    local_total = float(sum(step_ms))
    total_ms = max_over_ranks(local_total, dist, device)
    step_bytes = sum(c.kv_bytes for c in cases)
    value = whole_job_gbs(world, step_bytes, args.steps, total_ms)

    # roofline of the dominant kernel: the split-KV pass of the largest call
    big = max(range(len(cases)), key=lambda i: cases[i].kv_bytes)
    main_us = 1e3 * float(np.mean(main_ms[big]))
    achieved = cases[big].kv_bytes / (main_us * 1e-6) / 1e9
    traffic = ncu_traffic("splitkv.cuh", cases[big].p.name)
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": traffic, "kernel": "splitkv_kernel",
                "launch": cases[big].p.name, "peak_source": peak_src,
                "algorithmic_bytes_per_launch": cases[big].kv_bytes}
    points = []
    for c, cm, mm, om in zip(cases, call_ms, main_ms, outer_ms):
        us = 1e3 * statistics.mean(cm)
        points.append({"name": c.p.name, "us": round(us, 2),
                       "us_median": round(1e3 * statistics.median(cm), 2),
                       "us_p10": round(1e3 * float(np.percentile(cm, 10)), 2),
                       "us_p90": round(1e3 * float(np.percentile(cm, 90)), 2),
                       "main_kernel_us": round(1e3 * statistics.mean(mm), 2),
                       "outer_us": round(1e3 * statistics.mean(om), 2),
                       "kv_gbs": round(c.kv_bytes / (us * 1e-6) / 1e9, 1),
                       "frac_hbm": round(c.kv_bytes / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
                       "splits": c.info["splits"], "ctas": c.info["ctas"]})
    launches = sum(c.info["launches"] for c in cases) * args.steps

    if args.no_e2e:
        e2e_ms, h2d, d2h = [float("nan")], 0, 0
    else:
        e2e_ms, h2d, d2h = time_e2e(sdpa, cases, max(3, args.steps // 4), 2, device)
    e2e_val = step_bytes / (float(np.mean(e2e_ms)) * 1e-3) / 1e9 * world
    del cases
    torch.cuda.empty_cache()

    extra = {}
    if not args.no_secondary:
        sec_steps = max(3, min(args.steps, 20))
        gr = not args.eager
        # the 32K causal call runs last: seconds of full tensor load lower the
        # clock under the power cap for a while, which would slow the calls
        # timed right after it
        win = I.window_problems()
        extra["prefill"] = secondary(sdpa, win[:3] + I.encoder_problems() + win[3:], sec_steps,
                                     3, flush, sync_all, device, peaks, "tflops", gr, stream=True)
        time.sleep(1.0)
        # the verify sweep checks monotonicity in L between calls whose times
        # differ by about a microsecond: 60 samples per call (cheap at ~40 us)
        extra["verify"] = secondary(sdpa, I.verify_problems(), max(sec_steps, 60), 3, flush,
                                    sync_all, device, peaks, "tflops", gr, stream=True)
        extra["verify_checks"] = verify_checks(extra["verify"])
        extra["tiny"] = secondary(sdpa, [I.tiny_problem()], sec_steps, 3, flush, sync_all,
                                  device, peaks, "tflops", gr)
        extra["wide"] = secondary(sdpa, I.wide_problems(), sec_steps, 3, flush, sync_all,
                                  device, peaks, "tflops", gr)

    line = {"metric": METRIC, "value": round(value, 2), "unit": "GB/s (KV, decode)",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total_ms / args.steps, 4),
            "calls_timed_alone_ms_per_step": round(calls_sum_ms, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic N(0,1), seeded (no model weights)", "config": workload,
            "roofline": roofline, "clocks": clocks, "gpu_launches": launches,
            "e2e": {"value": round(e2e_val, 2), "unit": "GB/s (KV, decode)",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": round(float(np.mean(e2e_ms)), 3)},
            "points": points}
    line.update(extra)
    if extra:
        # compact per-call figures last on the line (prefill at the very end),
        # so that a reader who keeps only the end of the output still sees
        # every call: [name, path, us alone, fraction of the call's own
        # roofline, and for prefill and verify us back to back, its fraction]
        def brief(rows):
            return [[d["name"], d["path"], round(d["us"], 1), round(d["frac_roofline"], 3)] +
                    ([round(d["us_stream"], 1), round(d["frac_roofline_stream"], 3)]
                     if "us_stream" in d else []) for d in rows]
        line["summary"] = {
            "decode": [[d["name"], round(d["us"], 1), round(d["frac_hbm"], 3)] for d in points],
            "verify": brief(extra["verify"]), "verify_checks": extra["verify_checks"],
            "tiny": brief(extra["tiny"]), "wide": brief(extra["wide"]),
            "prefill": brief(extra["prefill"])}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        host_cases = [HostCase(p) for p in I.decode_problems()]
        val, secs, cores, calls = oracle_sample(host_cases, budget_s=10.0)
        line["cpu_baseline"] = {"value": round(val, 4), "unit": "GB/s (KV, decode)",
                                "cores": cores, "kind": "oracle",
                                "sample": f"{calls} decode calls of the sweep ({secs:.1f} s, fp64)"}
    if "summary" in line:
        line["summary"] = line.pop("summary")
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
