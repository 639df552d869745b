"""Benchmark of the mHC pre-map + post-map hot path (HC = 4) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload large] [--impl ours|reference]

One step = one mhc_pre (norm, projection, gates, Sinkhorn, aggregate) plus one mhc_post over one
batch of the workload (default: T=8192 tokens, H=7168, bf16; seeded synthetic inputs). The inputs
(R = 470 MB) are larger than the 126 MB L2, so no flush is needed between steps. Each rank runs
its own token shard (weak scaling, no data-path collective); rank 0 prints one JSON line with the
whole-job tokens/s taken over the slowest rank.

--impl reference times the fp64 CPU oracle (the only other implementation of this method here) on
a bounded sample of the same workload, on this host's cores.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "mHC pre+post tokens/s and HBM GB/s (% of roofline), T=8192 H=7168 bf16"
UNIT = "tokens/s"


def pre_bytes(T, H):
    """Algorithmic bytes of one pre-map call: R (8H) + y (2H) + pre/post/comb (96) per token, plus
    hc_fn (4H x 24 fp32) and scale/base once."""
    return T * (8 * H + 2 * H + 96) + 4 * H * 24 * 4 + 12 + 96


def post_bytes(T, H):
    """Algorithmic bytes of one post-map call: R (8H) + x (2H) + out (8H) + post/comb (80) per token."""
    return T * (18 * H + 80)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi sampling during the timed region (median SM clock, throttle reasons)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
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
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sms, maxs, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sms.append(float(parts[1]))
                maxs = max(maxs, float(parts[2]))
            except ValueError:
                continue
            for name, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sms:
            return None
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": maxs,
                "reasons": sorted(reasons), "samples": len(sms)}


def oracle_sample(w, n_tokens):
    """Time the fp64 oracle (pre + post) on the first n_tokens tokens of the workload."""
    import oracle
    R, x = w.R[:n_tokens], w.x[:n_tokens]
    t0 = time.perf_counter()
    r = oracle.pre(R, w.hc_fn, w.hc_scale, w.hc_base, rms_eps=w.rms_eps, pre_eps=w.pre_eps,
                   post_mult=w.post_mult, iters=w.iters, eps=w.eps)
    oracle.post(x, R, r["post"].astype(np.float32), r["comb"].astype(np.float32))
    dt = time.perf_counter() - t0
    return n_tokens / dt, dt, oracle.threads()


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def cpu_baseline(w, budget_s=12.0, max_passes=50):
    """Bounded sample: calibrate on a few tokens, then time about budget_s seconds of oracle work
    (the first n tokens, n <= T; when one pass over them takes less than budget_s, repeated
    passes until budget_s has elapsed), on all of the host's OpenMP threads and then on one."""
    import oracle

    def timed(budget):
        rate, _, _ = oracle_sample(w, 16)
        n = int(max(16, min(w.T, rate * budget)))
        tot, passes, cores = 0.0, 0, 1
        while passes < max_passes and (passes == 0 or tot < budget):
            _, dt, cores = oracle_sample(w, n)
            tot += dt
            passes += 1
        return n * passes / tot, n, passes, tot, cores

    all_threads = oracle.threads()
    v, n, passes, tot, cores = timed(budget_s)
    oracle.set_threads(1)
    try:
        v1, n1, p1, t1, _ = timed(budget_s / 3)
    finally:
        oracle.set_threads(all_threads)
    return {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"first {n} of {w.T} tokens (pre+post), {passes} pass(es), {tot:.1f} s",
            "value_1_thread": v1,
            "sample_1_thread": f"first {n1} of {w.T} tokens (pre+post), {p1} pass(es), {t1:.1f} s",
            "cpu_model": cpu_model()}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    from mhc_hyper_connection_02_b200 import inputs
    w = inputs.WORKLOADS[args.workload]()
    per_step = []
    base = None
    for i in range(args.warmup + args.steps):
        rate, dt, cores = oracle_sample(w, args.reference_tokens)
        if i >= args.warmup:
            per_step.append(dt)
        base = cores
    tot = sum(per_step)
    value = args.reference_tokens * len(per_step) / tot
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(per_step),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": f"{args.workload} T={w.T} H={w.H}", "tokens_per_step": args.reference_tokens},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": base, "kind": "oracle",
                         "sample": f"first {args.reference_tokens} of {w.T} tokens per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def load_traffic():
    """ncu DRAM bytes per launch recorded under profiles/, valid only for the kernel source they were
    taken from (sha256 of the library sources)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            return json.load(f)
    except Exception:
        return {}


# Source files that define each map's kernels (device code and launch configuration); a recorded
# DRAM traffic figure is used only while their digest matches the one it was recorded with.
KERNEL_SOURCES = {
    "post": ["mhc_post.cu", "mhc_device.cuh"],
    "pre": ["mhc_pre_tc.cu", "mhc_pre_cc.cu", "mhc_pre_fused.cu", "mhc_api.cu", "mhc_device.cuh"],
}


def source_digest(kernel):
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "mhc_hyper_connection_02_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def time_extras(mhc, R, x, out, y, pre, post, comb, hc_fn, scale, base, params, stream, T, H, dev,
                reps=10):
    """Device time of the entries beside the step, on the step's residual. Algorithmic bytes per
    token: pre from an external projection (one split): R (8H) + y (2H) + dot_mix (96) + sqrsum
    (4, external only) + pre/post/comb (96); expand: hidden (2H) + streams (8H); head_mean: R (8H)
    + y (2H); weighted head: R (8H) + y (2H) + weights (16), plus hc_fn (4H x 16) once; post with
    the next projection: the post-map's 18H + 80 plus S x 100 of partials; layer chain (that, then
    the next pre-map from the partials): the post-map's bytes plus the pre-map's 10H + 96;
    post-map backward: d_out (8H) + x (2H) + R (8H) + d_x (2H) + d_R (8H) + 160; pre-map backward:
    R (8H) + d_y (2H) + d_R (8H) + 96 of coefficient gradients, plus hc_fn and d_hc_fn once."""
    import torch
    g = torch.Generator(device=dev).manual_seed(5)
    dot = torch.randn((1, T, 24), generator=g, device=dev) * 0.01
    sq = torch.full((1, T), float(4 * H), device=dev)
    calls = {
        "pre_big_fuse": (lambda: mhc.pre_big_fuse(dot, sq, R, scale, base, 4 * H, y=y, pre=pre,
                                                  post=post, comb=comb, params=params,
                                                  stream=stream), T * (10 * H + 196)),
        "pre_big_fuse_with_prenorm": (lambda: mhc.pre_big_fuse_with_prenorm(
            dot[0], R, scale, base, y=y, pre=pre, post=post, comb=comb, params=params,
            stream=stream), T * (10 * H + 192)),
    }
    hidden = y  # a [T,H] bf16 row buffer of the step
    streams = torch.empty_like(R)
    fn4 = torch.randn((4 * H, 4), generator=g, device=dev) * 0.02
    s1 = torch.ones(1, device=dev)
    b4 = torch.zeros(4, device=dev)
    wts = torch.empty((T, 4), device=dev)
    hws = torch.empty(mhc.head_workspace_bytes(T, H), dtype=torch.uint8, device=dev)
    calls["expand"] = (lambda: mhc.expand(hidden, streams=streams, stream=stream), T * 10 * H)
    calls["head_mean"] = (lambda: mhc.head_mean(R, y=hidden, stream=stream), T * 10 * H)
    calls["head"] = (lambda: mhc.head(R, fn4, s1, b4, y=hidden, weights=wts, workspace=hws,
                                      stream=stream), T * (10 * H + 16) + 4 * H * 16)
    S = mhc.post_project_splits(T, H)
    if S > 0:
        pdm = torch.empty((S, T, 24), device=dev)
        psq = torch.empty((S, T), device=dev)
        wsp = torch.empty(max(1, int(mhc.lib().mhc_post_project_workspace_bytes(T, H))),
                          dtype=torch.uint8, device=dev)
        pre2, post2 = torch.empty_like(pre), torch.empty_like(post)
        comb2 = torch.empty_like(comb)

        def post_project():
            mhc.post_project(x, R, post, comb, hc_fn, out=out, dot_mix=pdm, sqrsum=psq,
                             workspace=wsp, stream=stream)

        def layer_chain():  # post of this site + the next site's pre-map on its output
            post_project()
            mhc.pre_big_fuse(pdm, psq, out, scale, base, 4 * H, num_splits=S, y=y, pre=pre2,
                             post=post2, comb=comb2, params=params, stream=stream)

        calls["post_project"] = (post_project, T * (18 * H + 80 + S * 100) + 4 * H * 96)
        calls["layer_chain"] = (layer_chain, T * (18 * H + 80) + T * (10 * H + 96) + 4 * H * 96)
    # Backward passes on the step's tensors: d_out / d_y random bf16, upstream coefficient grads.
    d_out = (torch.randn(R.shape, generator=g, device=dev) * 0.1).to(torch.bfloat16)
    d_y = d_out[:, 0, :].contiguous()
    d_c = torch.randn((T, 24), generator=g, device=dev) * 0.1
    d_pre_u, d_post_u = d_c[:, 0:4].contiguous(), d_c[:, 4:8].contiguous()
    d_comb_u = d_c[:, 8:24].contiguous()
    bws = torch.empty(int(mhc.lib().mhc_pre_backward_workspace_bytes(T, H)), dtype=torch.uint8,
                      device=dev)
    calls["post_backward"] = (lambda: mhc.post_backward(d_out, x, R, post, comb, stream=stream),
                              T * (28 * H + 160))
    calls["pre_backward"] = (lambda: mhc.pre_backward(
        R, hc_fn, scale, base, d_y=d_y, d_pre=d_pre_u, d_post=d_post_u, d_comb=d_comb_u,
        params=params, workspace=bws, stream=stream), T * (18 * H + 96) + 4 * H * 96 * 2)
    res = {}
    for name, (fn, nbytes) in calls.items():
        for _ in range(3):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        us = a.elapsed_time(b) / reps * 1e3
        res[name] = {"us": us, "algo_bytes": nbytes, "GBps": nbytes / us / 1e3,
                     "tokens_per_s": T / (us / 1e6)}
    assert mhc.device_status() == 0
    return res


def time_configs(mhc, inputs, dev, stream, reps=20):
    """Per-call device time of the other workloads (small, post4k, decode T in {1,4,16,32}, tail),
    each call timed alone with CUDA events. "flushed": a 256 MB buffer is written between calls
    (outside the timed region) so no input is left in the 126 MB L2; "warm": no flush, inputs (and
    for decode, hc_fn) L2-resident. Each call is queued behind a ~1 ms spin kernel so that the
    host's time to issue it is not inside the events (device time; CUDA graphs remove that host
    time in a serving loop). Returns {workload: {...}}."""
    import torch
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def dev_bf16(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)

    def timed(fn, flushed):
        fn()
        ts = []
        for _ in range(reps):
            if flushed:
                flush.fill_(1)
            # Queue the call behind ~1 ms of spinning so that the host's time to issue it (Python,
            # argument checks, launches) is not inside the events: device time only.
            torch.cuda._sleep(2000000)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) * 1e3)
        return statistics.median(ts)

    def graph_timed(call, n=10, reps=10):
        """Device time per call when n calls replay from one CUDA graph (a serving loop's setting:
        no per-call launch or event overhead), queued behind the spin like timed()."""
        gs = torch.cuda.Stream(dev)
        gs.wait_stream(stream)
        with torch.cuda.stream(gs):
            call(gs)  # first-call setup outside the capture
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=gs):
            for _ in range(n):
                call(gs)
        ts = []
        for _ in range(reps):
            torch.cuda._sleep(2000000)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) * 1e3 / n)
        del g
        return statistics.median(ts)

    def one(w, do_pre=True):
        R, x = dev_bf16(w.R), dev_bf16(w.x)
        W, sc, bs = (torch.from_numpy(a).to(dev) for a in (w.hc_fn, w.hc_scale, w.hc_base))
        prm = mhc.make_params(iters=w.iters, eps=w.eps, rms_eps=w.rms_eps, pre_eps=w.pre_eps,
                              post_mult=w.post_mult)
        ws = torch.empty(max(1, mhc.workspace_bytes(w.T, w.H)), dtype=torch.uint8, device=dev)
        y, pre, post, comb = mhc.pre(R, W, sc, bs, workspace=ws, params=prm, stream=stream)
        out = torch.empty_like(R)
        rec = {"T": w.T, "H": w.H}
        fp = lambda: mhc.pre(R, W, sc, bs, y=y, pre=pre, post=post, comb=comb, workspace=ws,
                             params=prm, stream=stream)
        fq = lambda: mhc.post(x, R, post, comb, out=out, stream=stream)
        for flushed in (True, False):
            tag = "flushed" if flushed else "warm"
            if do_pre:
                us = timed(fp, flushed)
                rec[f"pre_us_{tag}"] = us
                rec[f"pre_GBps_{tag}"] = pre_bytes(w.T, w.H) / us / 1e3
            us = timed(fq, flushed)
            rec[f"post_us_{tag}"] = us
            rec[f"post_GBps_{tag}"] = post_bytes(w.T, w.H) / us / 1e3
        if w.T <= 64:  # latency-bound shapes: also per call from a replayed CUDA graph
            if do_pre:
                rec["pre_us_graph"] = graph_timed(
                    lambda st: mhc.pre(R, W, sc, bs, y=y, pre=pre, post=post, comb=comb,
                                       workspace=ws, params=prm, stream=st))
            rec["post_us_graph"] = graph_timed(
                lambda st: mhc.post(x, R, post, comb, out=out, stream=st))
        return rec

    res = {"small": one(inputs.small()), "post4k": one(inputs.post4k(), do_pre=False),
           "tail": one(inputs.tail())}
    # What the event-timed method reports for one trivial kernel: a floor under every *_us figure
    # above (launch and event timestamp latency), not time spent in the library's kernels.
    tiny = torch.empty(1, device=dev)
    res["event_floor_us"] = timed(lambda: tiny.add_(1), False)
    for T in (1, 4, 16, 32):
        res[f"decode_T{T}"] = one(inputs.decode(T))
    assert mhc.device_status() == 0
    del flush
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="large", choices=["large", "post4k", "small", "tail", "decode"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--reference-tokens", type=int, default=256)
    ap.add_argument("--pre-path", type=int, default=0)
    ap.add_argument("--post-path", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--only", default="both", choices=["both", "pre", "post"],
                    help="time one map only (profiling); the JSON line is for the full step")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the workload's token count (profiling smaller cases)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip timing the entries beside the step and the other workloads")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist
    import mhc_hyper_connection_02_b200 as mhc
    from mhc_hyper_connection_02_b200 import inputs
    from mhc_hyper_connection_02_b200.shard import global_max, throughput

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    if ws > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    w = inputs.WORKLOADS[args.workload](T=args.tokens) if args.tokens else inputs.WORKLOADS[args.workload]()
    T, H = w.T, w.H
    dev = torch.device("cuda", local)
    R = torch.from_numpy(w.R.view(np.int16)).view(torch.bfloat16).to(dev)
    x = torch.from_numpy(w.x.view(np.int16)).view(torch.bfloat16).to(dev)
    hc_fn = torch.from_numpy(w.hc_fn).to(dev)
    scale = torch.from_numpy(w.hc_scale).to(dev)
    base = torch.from_numpy(w.hc_base).to(dev)
    y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    pre = torch.empty((T, 4), dtype=torch.float32, device=dev)
    post = torch.empty((T, 4), dtype=torch.float32, device=dev)
    comb = torch.empty((T, 4, 4), dtype=torch.float32, device=dev)
    out = torch.empty_like(R)
    ws_bytes = mhc.workspace_bytes(T, H)
    workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    params = mhc.make_params(iters=w.iters, eps=w.eps, rms_eps=w.rms_eps, pre_eps=w.pre_eps,
                             post_mult=w.post_mult)
    stream = torch.cuda.current_stream(dev)

    do_pre, do_post = args.only in ("both", "pre"), args.only in ("both", "post")

    def step():
        if do_pre:
            mhc.pre(R, hc_fn, scale, base, y=y, pre=pre, post=post, comb=comb, workspace=workspace,
                    params=params, path=args.pre_path, stream=stream)
        if do_post:
            mhc.post(x, R, post, comb, out=out, path=args.post_path, stream=stream)

    if not do_pre:  # post-only timing still needs valid coefficients
        mhc.pre(R, hc_fn, scale, base, y=y, pre=pre, post=post, comb=comb, workspace=workspace,
                params=params, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert mhc.device_status() == 0

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = mhc.launch_count()
    # A spin kernel ahead of the start event lets the host queue the steps before the device
    # reaches them: the first step then does not include the host's enqueue latency after the
    # synchronize (the device work timed is the same).
    with torch.cuda.stream(stream):
        torch.cuda._sleep(4000000)
    start.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        if do_pre:
            mhc.pre(R, hc_fn, scale, base, y=y, pre=pre, post=post, comb=comb,
                    workspace=workspace, params=params, path=args.pre_path, stream=stream)
        ev[i][1].record(stream)
        if do_post:
            mhc.post(x, R, post, comb, out=out, path=args.post_path, stream=stream)
        ev[i][2].record(stream)
    stop.record(stream)
    torch.cuda.synchronize()
    launches = mhc.launch_count() - launches0
    if ws > 1:
        dist.barrier()
    clocks = sampler.stop()
    assert mhc.device_status() == 0

    total_ms = start.elapsed_time(stop)
    pre_ms = [a.elapsed_time(b) for a, b, _ in ev]
    post_ms = [b.elapsed_time(c) for _, b, c in ev]
    max_ms = global_max(total_ms, device=dev)

    # End to end through the public API with host buffers: every step copies its inputs from
    # pinned host memory (R, x and the weights), runs the two calls and reads its results back (out,
    # y, pre, post, comb), all inside the timed region. Steps are pipelined over two device buffer
    # sets and three streams: step i's host-to-device copies overlap step i-1's kernels and step
    # i-2's device-to-host copies (PCIe is full duplex).
    e2e = None
    if not args.no_e2e and args.only == "both":
        hR = torch.from_numpy(w.R.view(np.int16)).view(torch.bfloat16).pin_memory()
        hx = torch.from_numpy(w.x.view(np.int16)).view(torch.bfloat16).pin_memory()
        hW = torch.from_numpy(w.hc_fn).pin_memory()
        hs = torch.from_numpy(w.hc_scale).pin_memory()
        hb = torch.from_numpy(w.hc_base).pin_memory()
        slots = []
        for _ in range(2):
            d = {"R": torch.empty_like(R), "x": torch.empty_like(x),
                 "W": torch.empty_like(hc_fn), "s": torch.empty_like(scale),
                 "b": torch.empty_like(base), "y": torch.empty_like(y),
                 "pre": torch.empty_like(pre), "post": torch.empty_like(post),
                 "comb": torch.empty_like(comb), "out": torch.empty_like(out),
                 "ws": torch.empty_like(workspace)}
            h = {"out": torch.empty(out.shape, dtype=torch.bfloat16).pin_memory(),
                 "y": torch.empty(y.shape, dtype=torch.bfloat16).pin_memory(),
                 "pre": torch.empty((T, 4), dtype=torch.float32).pin_memory(),
                 "post": torch.empty((T, 4), dtype=torch.float32).pin_memory(),
                 "comb": torch.empty((T, 4, 4), dtype=torch.float32).pin_memory()}
            ev = {k: torch.cuda.Event() for k in ("in", "comp", "out")}
            slots.append((d, h, ev))
        h2d = sum(a.numel() * a.element_size() for a in (hR, hx, hW, hs, hb))
        d2h = sum(a.numel() * a.element_size() for a in slots[0][1].values())
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def e2e_run(nsteps):
            s_in.wait_stream(stream)
            s_out.wait_stream(stream)
            for i in range(nsteps):
                d, h, ev = slots[i % 2]
                if i >= 2:
                    s_in.wait_event(ev["comp"])  # step i-2's kernels are done with this slot
                with torch.cuda.stream(s_in):
                    for k, src in (("R", hR), ("x", hx), ("W", hW), ("s", hs), ("b", hb)):
                        d[k].copy_(src, non_blocking=True)
                    ev["in"].record(s_in)
                stream.wait_event(ev["in"])
                if i >= 2:
                    stream.wait_event(ev["out"])  # step i-2's results have left this slot
                mhc.pre(d["R"], d["W"], d["s"], d["b"], y=d["y"], pre=d["pre"], post=d["post"],
                        comb=d["comb"], workspace=d["ws"], params=params, stream=stream)
                mhc.post(d["x"], d["R"], d["post"], d["comb"], out=d["out"], stream=stream)
                ev["comp"].record(stream)
                s_out.wait_event(ev["comp"])
                with torch.cuda.stream(s_out):
                    for k in ("out", "y", "pre", "post", "comb"):
                        h[k].copy_(d[k], non_blocking=True)
                    ev["out"].record(s_out)
            stream.wait_stream(s_in)
            stream.wait_stream(s_out)

        e2e_steps = max(4, min(args.steps, 10))
        e2e_run(2)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        e2e_run(e2e_steps)
        b.record(stream)
        torch.cuda.synchronize()
        assert torch.equal(slots[(e2e_steps - 1) % 2][1]["out"].view(torch.int16).view(-1)[:64],
                           out.view(torch.int16).view(-1)[:64].cpu())
        e2e = {"value": throughput(T, ws, e2e_steps, global_max(a.elapsed_time(b), device=dev)),
               "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "pipelined": "2 buffer sets, H2D / kernels / D2H on three streams"}

    configs = None
    if not args.no_extras and args.only == "both" and args.workload == "large":
        configs = time_configs(mhc, inputs, dev, stream)
    extras = None
    if not args.no_extras and args.only == "both":
        extras = time_extras(mhc, R, x, out, y, pre, post, comb, hc_fn, scale, base, params,
                             stream, T, H, dev)

    if rank == 0:
        hbm, tflops, peak_src = load_peaks()
        post_avg_s = statistics.mean(post_ms) / 1e3
        pre_avg_s = statistics.mean(pre_ms) / 1e3
        pb, qb = post_bytes(T, H), pre_bytes(T, H)
        post_gbs = pb / post_avg_s / 1e9 if do_post else 0.0
        pre_gbs = qb / pre_avg_s / 1e9 if do_pre else 0.0
        # The roofline object describes one kernel: the post-map is a single launch and the
        # longest kernel of the step (the split pre-map is a chain of four shorter launches,
        # reported as a whole call under "kernels").
        dominant = "post" if do_post else "pre"
        traffic_rec = load_traffic().get(f"{dominant}:{args.workload}")
        traffic = None
        if traffic_rec and traffic_rec.get("source") == source_digest(dominant):
            traffic = traffic_rec.get("bytes_per_launch")
        ach = post_gbs if dominant == "post" else pre_gbs
        line = {
            "metric": METRIC,
            "value": throughput(T, ws, args.steps, max_ms),
            "unit": UNIT, "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": max_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{args.workload}: T={T} H={H} HC=4 bf16, seeded synthetic",
                       "tokens_per_gpu": T, "hidden": H, "sinkhorn_iters": w.iters,
                       "parallelism": f"token shards x{ws}, no collective",
                       "l2": "inputs larger than L2 (R = %d MB)" % (T * 8 * H // 2 ** 20)},
            "roofline": {"bound": "hbm", "kernel": f"mhc_{dominant}", "achieved": ach,
                         "peak": hbm, "unit": "GB/s", "frac": ach / hbm, "traffic": traffic,
                         "peak_source": f"{peak_src} hbm_gbs (MEASURED_PEAKS.json)"},
            "kernels": {},
            "gpu_launches": int(launches),
            "clocks": clocks,
            "e2e": e2e,
        }
        if do_pre:
            # The pre-map's own roofline object: the whole call (its kernels chained by
            # programmatic dependent launch), algorithmic bytes over the call's event time.
            pre_traffic_rec = load_traffic().get(f"pre:{args.workload}")
            pre_traffic = None
            if pre_traffic_rec and pre_traffic_rec.get("source") == source_digest("pre"):
                pre_traffic = pre_traffic_rec.get("bytes_per_call")
            line["pre_roofline"] = {
                "bound": "hbm", "kernel": "mhc_pre (whole call)", "achieved": pre_gbs,
                "peak": hbm, "unit": "GB/s", "frac": pre_gbs / hbm, "traffic": pre_traffic,
                "peak_source": f"{peak_src} hbm_gbs (MEASURED_PEAKS.json)",
                "path": args.pre_path}
            line["kernels"]["pre"] = {
                "us": pre_avg_s * 1e6, "algo_bytes": qb, "GBps": pre_gbs,
                "frac_measured": pre_gbs / hbm, "frac_8TBps": pre_gbs / 8000.0,
                "path": args.pre_path}
        if do_post:
            line["kernels"]["post"] = {
                "us": post_avg_s * 1e6, "algo_bytes": pb, "GBps": post_gbs,
                "frac_measured": post_gbs / hbm, "frac_8TBps": post_gbs / 8000.0,
                "path": args.post_path}
        if extras:
            for v in extras.values():
                v["frac_measured"] = v["GBps"] / hbm
            line["extras"] = extras
        if configs:
            line["configs"] = configs
        if not args.no_cpu_baseline and ws == 1:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
