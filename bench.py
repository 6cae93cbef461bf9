#!/usr/bin/env python
"""Benchmark of the entropy-bound canvas sampler step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload: one 256 x 262144 bf16 canvas per GPU (the model card's canvas and
vocabulary), seeded synthetic decoder logits pre-generated for all 48 steps of
an entropy-bound trajectory (temperature 0.8 -> 0.4, entropy_bound 0.1,
adaptive stop 0.005 / 1 stable step).  A "step" is one eb_sampler_step call:
every logit of every active canvas read once, entropies, argmax, draws,
commit, renoise, stop test.  Each step reads its own 134 MB of logits, more
than the 126 MB L2, so no step hits in L2 on the previous one's data.

Timing: W eager warm-up steps, then timed regions of exactly K steps, each
with CUDA events on the launching stream between a barrier + synchronize on
both sides (max over ranks); the K steps are replayed from CUDA graphs (one
per full 48-step trajectory, one for the remaining prefix; each starts with
the canvas init kernel), and the median over the regions is reported.  A
step is one kernel launch, so the step kernel's average launch duration (for
the roofline) is the region's time over its K launches.  For N > 1 each rank
runs its own canvas (global canvas index = rank): no data-path collective,
weak scaling.

At N = 1 the other large workloads (serve 8x, br 4x, stress 32x fp32) are
timed afterwards as whole 48-step trajectories and reported under "configs",
with the sampler fused into the LM head (hidden size 2560, 1 and 8 canvases:
"lmhead", "lmhead8") and its unfused counterpart.

--impl reference times the CPU oracle (the float64 restatement in oracle/)
on the host cores, rank 0 only, on bounded samples of the same workload.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "canvas positions sampled/sec and HBM GB/s (% of B200 peak), 256x262144 bf16 step"
UNIT = "positions/s"
WORKLOAD = "canvas"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=9600)
    p.add_argument("--warmup", type=int, default=48)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--e2e-steps", type=int, default=48)
    p.add_argument("--repeats", type=int, default=0,
                   help="timed regions of exactly K steps (median reported); 0 = automatic")
    p.add_argument("--configs", default="all",
                   help="other workloads timed after the headline one: all, none, or a list "
                        "of serve,br,stress,lmhead,lmhead8 (N = 1 only by default)")
    p.add_argument("--split-v", action="store_true",
                   help="vocabulary-sharded canvas: each rank holds a slice of the vocabulary; "
                        "a step is the slice pass, one all-gather of the records, the combine")
    p.add_argument("--profile", action="store_true",
                   help="small case for ncu: logits of steps 0-2 only, three eager steps")
    p.add_argument("--profile-lmhead", action="store_true",
                   help="small case for ncu: three LM-head steps, 1 x 256 positions, "
                        "V = 32768, hidden size 2560")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def peak_label(kind, key, fallback):
    """Where a roofline peak came from."""
    if kind == "measured":
        return f"measured: MEASURED_PEAKS.json {key}"
    return f"fallback: {fallback}, an earlier B200 measurement (no MEASURED_PEAKS.json)"


def tensor_peak():
    """Dense bf16 tensor peak (TFLOP/s): the measured burst figure, else the
    pool's fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def run_lmhead_config(E, synth, dev, B, d, barrier, max_over_ranks):
    """The sampler fused into the LM head (eb_lmhead_step): 48-step
    trajectories from the hidden states of the synthetic recipe (hidden size
    d, an assumption: the pages give none), replayed from a CUDA graph; and,
    for context, the same steps unfused (cuBLAS bf16 GEMM to bf16 logits,
    then the sampler step)."""
    import torch

    from synth import lmhead as LM
    w = synth.WORKLOADS["canvas"].replace(B=B, seed=31)
    N = w.num_steps
    wc = LM.weight_codes(w.V, d, seed=w.seed)
    W = LM.to_bf16(wc).to(dev)
    hs = [LM.to_bf16(LM.hidden_codes(wc, w.B, w.L, s, N, seed=w.seed)).to(dev) for s in range(N)]
    del wc
    eb = E.EBSampler(w.B, w.L, w.V, device=dev, **w.sampler_config())
    canvas, committed, stop = eb.new_canvas()
    H, amax = eb.outputs()
    lg = torch.empty((w.B, w.L, w.V), dtype=torch.bfloat16, device=dev)

    def fused():
        eb.init_canvas(canvas, committed, stop)
        for s in range(N):
            eb.lmhead_step(hs[s], W, s, canvas, committed, H, amax, stop)

    def unfused():
        eb.init_canvas(canvas, committed, stop)
        for s in range(N):
            torch.matmul(hs[s], W.T, out=lg.view(w.B * w.L, w.V))
            eb.step(lg, s, canvas, committed, H, amax, stop)

    out = {}
    for name, fn in (("fused", fused), ("unfused", unfused)):
        fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            fn()
            torch.cuda.synchronize()
            with torch.cuda.graph(g, stream=side):
                fn()
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        times = timed_regions(g.replay, 5, barrier, torch.cuda.current_stream(dev))
        out[name] = max_over_ranks(statistics.median(times)) / N
        del g
    status = eb.status()
    eb.close()
    flop = 2.0 * w.B * w.L * w.V * d
    peak, kind = tensor_peak()
    tfl = flop / (out["fused"] * 1e-3) / 1e12
    return {
        "workload": f"{B} x 256 x 262144, hidden size {d} (bf16 hidden states and LM head), "
                    "logits formed and reduced on chip",
        "value": w.B * w.L / (out["fused"] * 1e-3), "unit": UNIT,
        "ms_per_step": out["fused"], "steps": N, "status": status,
        "unfused_ms_per_step": out["unfused"],
        "roofline": {"bound": "tensor", "achieved": tfl, "peak": peak, "unit": "TFLOP/s",
                     "frac": tfl / peak, "kernel": "ebk::lmhead_kernel<true>",
                     "flop_per_step": flop,
                     "peak_source": peak_label(kind, "bf16_tflops (cuBLAS burst)",
                                               f"{FALLBACK_BF16_TFLOPS:.0f} TFLOP/s")},
    }


def kernel_source_hash():
    h = hashlib.sha256()
    for f in ("eb_stream.cuh", "eb_finish.cuh", "eb_common.cuh", "eb_device.cuh", "eb_sampler.cu"):
        with open(os.path.join(ROOT, "entropy_bound_canvas_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per launch of the step kernel from the committed ncu summary,
    if it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "stream_kernel_canvas_1x256x262144_bf16.md")
    try:
        txt = open(path).read()
    except OSError:
        return None
    m1 = re.search(r"source_sha256_16:\s*([0-9a-f]{16})", txt)
    m2 = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", txt)
    if not m1 or not m2 or m1.group(1) != kernel_source_hash():
        return None
    return int(m2.group(1))


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        loaded = [x for x, p in zip(sm, power) if p > 200.0] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


# --------------------------------------------------------------------------- reference arm

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np

    import oracle as O
    import synth

    w = synth.WORKLOADS[WORKLOAD]
    cfg = O.Config(B=w.B, L=w.L, V=w.V, group_size=64, **w.sampler_config())
    # Per step: the oracle's full per-position work (entropy, argmax, two-level
    # draw) on ROWS positions of the canvas at that step, plus the canvas
    # decisions; bounded so the whole run ends within a few minutes.
    rows_per_step = 4
    K, W = args.steps, args.warmup
    total = K + W
    budget_rows = 12000  # ~2 minutes of rows at ~10 ms each
    if total * rows_per_step > budget_rows:
        rows_per_step = max(1, budget_rows // total)
    st = O.State(cfg).init()
    times = []
    cache = {}
    for i in range(total):
        s = i % w.num_steps
        l0 = (s * 37) % (w.L - rows_per_step + 1)
        if (s, l0) not in cache:
            cache[(s, l0)] = synth.generate_host(w, s, 0, 1, l0, rows_per_step)[0]
        rows = cache[(s, l0)]
        t0 = time.perf_counter()
        T = O.temperature(cfg, s)
        H = np.zeros(w.L)
        amax = np.zeros(w.L, np.int32)
        pm = np.zeros(w.L)
        smp = np.zeros(w.L, np.int32)
        for k in range(rows_per_step):
            l = l0 + k
            H[l], pm[l], amax[l], _ = O.row_stats(rows[k], 1.0 / T)
            if not st.committed[0, l]:
                smp[l] = O.sample(cfg, rows[k], 1.0 / T, 0, l, s)[0]
        O.canvas_decide(st, 0, s, H, amax, pm, smp)
        dt = time.perf_counter() - t0
        if st.stop[0] or s == w.num_steps - 1:
            st = O.State(cfg).init()
        if i >= W:
            times.append(dt)
    el = sum(times)
    value = K * rows_per_step / el
    sample = (f"{rows_per_step} of 256 positions per step (entropy, argmax and two-level draw "
              f"of each, 262144 bf16 logits) plus the canvas decisions; {K} timed steps")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": K, "warmup": W, "ms_per_step": 1e3 * el / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "canvas 1x256x262144 bf16 (oracle sample)", "B": 1, "L": 256,
                   "V": 262144},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- our arm

def host_info():
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_nproc": os.cpu_count(), "cpu_model": model}


def cpu_baseline(w, logits_steps, states):
    """The oracle, as it stands, on full canvas steps at a few step indices."""
    import numpy as np

    import oracle as O
    cfg = O.Config(B=w.B, L=w.L, V=w.V, group_size=64, **w.sampler_config())
    t_total, n_pos = 0.0, 0
    used = []
    for s, (cv, cm, prev) in states.items():
        st = O.State(cfg).init()
        st.canvas[0], st.committed[0], st.prev[0] = cv, cm, prev
        lg = logits_steps[s][0].view(__import__("torch").int16).cpu().numpy().view(np.uint16)
        t0 = time.perf_counter()
        O.step_canvas(st, 0, lg, s)
        t_total += time.perf_counter() - t0
        n_pos += w.L
        used.append(s)
    out = {"value": n_pos / t_total, "unit": UNIT, "cores": 1, "kind": "oracle",
           "sample": f"{len(used)} full 256-position canvas steps (s = {used[0]}, {used[1]}, ..., "
                     f"{used[-1]}) of the same trajectory "
                     f"(single thread, float64), {t_total:.1f} s of CPU work"}
    out.update(host_info())
    return out


class Trajectory:
    """One workload on one device: a sampler handle, its canvas buffers and
    the logits of every step resident in HBM (or `rotate` buffers reused
    round-robin when 48 steps of the workload do not fit)."""

    def __init__(self, E, synth, w, dev, rank, rotate=None):
        import torch
        self.w, self.dev = w, dev
        self.N = w.num_steps
        nbuf = self.N if rotate is None else rotate
        dt = torch.float32 if w.dtype == synth.F32 else torch.bfloat16
        self.logits = [torch.empty((w.B, w.L, w.V), dtype=dt, device=dev) for _ in range(nbuf)]
        for s in range(nbuf):
            synth.generate_device(w, s, self.logits[s], b0=rank * w.B)
        self.eb = E.EBSampler(w.B, w.L, w.V, device=dev, canvas_offset=rank * w.B,
                              **w.sampler_config())
        self.canvas, self.committed, self.stop = self.eb.new_canvas()
        self.H, self.amax = self.eb.outputs()
        self.graphs = {}

    def lg(self, s):
        return self.logits[s % len(self.logits)]

    def run(self, n):
        """init + the first n steps, on the current stream."""
        self.eb.init_canvas(self.canvas, self.committed, self.stop)
        for s in range(n):
            self.eb.step(self.lg(s), s, self.canvas, self.committed, self.H, self.amax, self.stop)

    def active_per_step(self):
        """Active canvases at the start of each step of one trajectory (untimed)."""
        import torch
        act = []
        self.eb.init_canvas(self.canvas, self.committed, self.stop)
        for s in range(self.N):
            act.append(int((self.stop == 0).sum().item()))
            self.eb.step(self.lg(s), s, self.canvas, self.committed, self.H, self.amax, self.stop)
        torch.cuda.synchronize()
        return act

    def graph(self, n):
        """A CUDA graph of init + the first n steps (captured once)."""
        import torch
        if n not in self.graphs:
            g = torch.cuda.CUDAGraph()
            side = torch.cuda.Stream(self.dev)
            side.wait_stream(torch.cuda.current_stream(self.dev))
            with torch.cuda.stream(side):
                self.run(n)
                torch.cuda.synchronize()
                with torch.cuda.graph(g, stream=side):
                    self.run(n)
            torch.cuda.synchronize()
            self.graphs[n] = g
        return self.graphs[n]

    def close(self):
        self.graphs.clear()
        self.eb.close()
        self.logits.clear()


def timed_regions(replay, repeats, barrier, stream):
    """Each region: barrier + synchronize, CUDA events around replay(),
    synchronize + barrier.  Returns the region times in ms."""
    import torch
    out = []
    for _ in range(repeats):
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        replay()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        out.append(e0.elapsed_time(e1))
    return out


def roofline_of(kernel, launches, bytes_total, region_ms, peak, peak_kind):
    """Step-kernel roofline of a timed region.  A step is one kernel launch
    (the stream kernel, canvas decisions included), so its average launch
    duration is the region's time over the launches in it; the region's few
    canvas-init launches (about 2 us each) are counted against it.
    Algorithmic bytes per launch: every logit of the canvases active at that
    step, once."""
    k_ms = region_ms / launches
    bytes_launch = bytes_total / launches
    achieved = bytes_launch / (k_ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "kernel": kernel, "kernel_ms": k_ms,
            "algorithmic_bytes": bytes_launch,
            "timing": "CUDA events around graph replays on the launching stream; "
                      "region time / step-kernel launches",
            "peak_source": peak_label(peak_kind, "hbm_gbs (copy)", f"{FALLBACK_HBM_GBS:.0f} GB/s")}


LMHEAD_D = 2560  # hidden size of the LM-head configs (the pages give none)

EXTRA = {
    # name -> (rotate buffers or None, description)
    "serve": (None, "8 x 256 x 262144 bf16 per GPU, staggered stops, 48 steps resident"),
    "br": (None, "4 x 256 x 262144 bf16 per GPU, block refinement, greedy, 48 steps resident"),
    "stress": (3, "32 x 256 x 262144 fp32 per GPU, Zipf-like logits, 3 step buffers "
                  "rotated (8.6 GB each)"),
}


def run_ours(args):
    import torch

    import entropy_bound_canvas_b200 as E
    import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    def max_over_ranks(x):
        if dist is None:
            return x
        t = torch.tensor([x], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def sum_over_ranks(x):
        if dist is None:
            return x
        t = torch.tensor([x], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
        return float(t.item())

    w = synth.WORKLOADS[WORKLOAD]
    N = w.num_steps
    K, W = args.steps, max(3, args.warmup)
    stream = torch.cuda.current_stream(dev)
    peak, peak_kind = peaks()

    tr = Trajectory(E, synth, w, dev, rank)
    torch.cuda.synchronize()

    # reference trajectory (untimed): active canvases per step, snapshots for the CPU baseline
    active = []
    snaps = {}
    tr.eb.init_canvas(tr.canvas, tr.committed, tr.stop)
    for s in range(N):
        active.append(int((tr.stop == 0).sum().item()))
        if s % 2 == 0:  # 24 of the 48 steps: about 15 s of oracle work
            snaps[s] = (tr.canvas[0].cpu().numpy().copy(), tr.committed[0].cpu().numpy().copy(),
                        tr.amax[0].cpu().numpy().copy())
        tr.eb.step(tr.lg(s), s, tr.canvas, tr.committed, tr.H, tr.amax, tr.stop)
    torch.cuda.synchronize()
    stop_step = next((s for s in range(N) if s + 1 < N and active[s + 1] == 0), N - 1)

    # warm-up: W eager steps along the trajectory
    tr.eb.init_canvas(tr.canvas, tr.committed, tr.stop)
    for i in range(W):
        s = i % N
        if s == 0 and i > 0:
            tr.eb.init_canvas(tr.canvas, tr.committed, tr.stop)
        tr.eb.step(tr.lg(s), s, tr.canvas, tr.committed, tr.H, tr.amax, tr.stop)
    torch.cuda.synchronize()

    # exactly K steps per timed region: full trajectories and a prefix, each
    # from a CUDA graph (init + steps), replayed back to back
    full, rem = divmod(K, N)
    g_full = tr.graph(N) if full else None
    g_rem = tr.graph(rem) if rem else None
    for _ in range(2):  # warm the graphs
        if g_full is not None:
            g_full.replay()
        if g_rem is not None:
            g_rem.replay()
    torch.cuda.synchronize()

    def region():
        for _ in range(full):
            g_full.replay()
        if g_rem is not None:
            g_rem.replay()

    # one kernel per step, one init kernel per graph
    launches = full * (N + 1) + ((rem + 1) if rem else 0)
    positions = full * sum(active) * w.L + sum(active[:rem]) * w.L
    bytes_total = (full * sum(active) + sum(active[:rem])) * w.L * w.V * w.elt
    repeats = args.repeats or max(3, min(50, int(0.5 / max(1e-5, K * 40e-6))))

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    times = timed_regions(region, repeats, barrier, stream)
    clk = clocks.stop()
    el_ms = max_over_ranks(statistics.median(times))
    positions_all = sum_over_ranks(float(positions))
    bytes_all = sum_over_ranks(float(bytes_total))
    value = positions_all / (el_ms * 1e-3)
    hbm_gbs_job = bytes_all / (el_ms * 1e-3) / 1e9

    # full-trajectory step time (48 steps) for reference, when the timed region is shorter
    traj_ms = None
    if full == 0:
        g48 = tr.graph(N)
        traj = timed_regions(g48.replay, 3, barrier, stream)
        traj_ms = max_over_ranks(statistics.median(traj)) / N

    kname = f"ebk::stream_kernel<{'f32' if w.elt == 4 else 'bf16'}>"
    roof = roofline_of(kname, K, bytes_total, el_ms, peak, peak_kind)
    roof["traffic"] = recorded_traffic()

    # end-to-end: host (pinned) logits -> device, step, result back to host, every step
    e2e = None
    if not args.no_e2e:
        n_e2e = min(args.e2e_steps, N)
        host = [tr.lg(s).cpu().pin_memory() for s in range(n_e2e)]
        dev_buf = torch.empty_like(tr.lg(0))
        out_cv = torch.empty((w.B, w.L), dtype=torch.int32).pin_memory()
        out_cm = torch.empty((w.B, w.L), dtype=torch.uint8).pin_memory()
        out_sp = torch.empty((w.B,), dtype=torch.uint8).pin_memory()
        tr.eb.init_canvas(tr.canvas, tr.committed, tr.stop)
        torch.cuda.synchronize()
        barrier()
        t0 = time.perf_counter()
        x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        x0.record(stream)
        pos_e2e = 0
        for s in range(n_e2e):
            dev_buf.copy_(host[s], non_blocking=True)
            tr.eb.step(dev_buf, s, tr.canvas, tr.committed, tr.H, tr.amax, tr.stop)
            out_cv.copy_(tr.canvas, non_blocking=True)
            out_cm.copy_(tr.committed, non_blocking=True)
            out_sp.copy_(tr.stop, non_blocking=True)
            stream.synchronize()
            pos_e2e += active[s] * w.L
        x1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(x0.elapsed_time(x1))
        pos_e2e = sum_over_ranks(float(pos_e2e))
        e2e = {"value": pos_e2e / (e2e_ms * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": w.B * w.L * w.V * w.elt,
               "d2h_bytes_per_step": w.B * w.L * 4 + w.B * w.L + w.B,
               "steps": n_e2e, "wall_s": time.perf_counter() - t0}
        del host

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, tr.logits, snaps)
    tr.close()
    del tr
    torch.cuda.empty_cache()

    # the other large workloads: full 48-step trajectories from one graph each
    extra = {}
    names = [] if args.configs == "none" else (
        list(EXTRA) + ["lmhead", "lmhead8"] if args.configs == "all"
        else args.configs.split(","))
    if world > 1 and args.configs == "all":
        names = []  # the scaling runs time the headline workload only
    for name in names:
        if name.startswith("lmhead"):
            Bx = 8 if name == "lmhead8" else 1
            extra[name] = run_lmhead_config(E, synth, dev, Bx, LMHEAD_D, barrier, max_over_ranks)
            torch.cuda.empty_cache()
            continue
        rotate, desc = EXTRA[name]
        wx = synth.WORKLOADS[name]
        tx = Trajectory(E, synth, wx, dev, rank, rotate=rotate)
        act = tx.active_per_step()
        gx = tx.graph(wx.num_steps)
        gx.replay()
        torch.cuda.synchronize()
        tx_times = timed_regions(gx.replay, 5, barrier, stream)
        ms = max_over_ranks(statistics.median(tx_times))
        pos = sum_over_ranks(float(sum(act) * wx.L))
        byt = sum_over_ranks(float(sum(act) * wx.L * wx.V * wx.elt))
        rf = roofline_of("", wx.num_steps, sum(act) * wx.L * wx.V * wx.elt, ms, peak, peak_kind)
        gbs = byt / (ms * 1e-3) / 1e9
        extra[name] = {
            "workload": desc, "value": pos / (ms * 1e-3), "unit": UNIT,
            "ms_per_step": ms / wx.num_steps, "steps": wx.num_steps, "repeats": len(tx_times),
            "active_canvases_per_step": act, "dtype": "f32" if wx.elt == 4 else "bf16",
            "hbm_gbs": gbs, "hbm_frac_of_peak": gbs / (peak * world),
            "roofline": {k: rf[k] for k in ("achieved", "frac", "kernel_ms", "algorithmic_bytes")},
        }
        tx.close()
        del tx, gx
        torch.cuda.empty_cache()

    if rank == 0:
        timing = (f"each timed region is exactly {K} steps replayed from CUDA graphs "
                  f"({full} full 48-step trajectories + a {rem}-step prefix, one init kernel "
                  f"each); {repeats} regions, median reported")
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": el_ms / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {
                "workload": "canvas 1x256x262144 bf16 per GPU, 48-step entropy-bound trajectory",
                "B_per_gpu": w.B, "L": w.L, "V": w.V, "num_steps": N, "seed": w.seed,
                "stop_step": stop_step, "repeats": repeats,
                "l2": "inputs larger than L2: each step reads its own 134 MB of logits",
                "timing": timing,
            },
            "hbm_gbs": hbm_gbs_job,
            "hbm_frac_of_peak": hbm_gbs_job / (peak * world),
            "trajectory_ms_per_step": traj_ms,
            "region_ms": {"median": statistics.median(times), "min": min(times),
                          "max": max(times)},
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk,
            "configs": extra,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def run_split_v(args):
    """The canvas workload with its vocabulary split over the ranks (a
    tensor-parallel LM head): rank r holds a contiguous, group-aligned slice
    of every row; each step runs the slice pass on every rank, one NCCL
    all-gather of the per-position records and the combine.  Total work is
    fixed, so this is strong scaling.  Eager steps (the collective is not
    captured), timed with CUDA events between barriers, max over ranks."""
    import torch

    import entropy_bound_canvas_b200 as E
    import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    w = synth.WORKLOADS[WORKLOAD]
    N = w.num_steps
    K, W = args.steps, max(3, args.warmup)
    ng = (w.V + 63) // 64
    per = (ng + world - 1) // world
    lo, hi = min(ng, rank * per) * 64, min(w.V, min(ng, (rank + 1) * per) * 64)
    full = torch.empty((w.B, w.L, w.V), dtype=torch.bfloat16, device=dev)
    sl = []
    for s in range(N):
        synth.generate_device(w, s, full)
        sl.append(full[:, :, lo:hi].contiguous())
    del full
    torch.cuda.empty_cache()
    eb = E.EBSampler(w.B, w.L, hi - lo, device=dev, vocab_offset=lo, vocab_total=w.V,
                     **w.sampler_config())
    canvas, committed, stop = eb.new_canvas()
    H, amax = eb.outputs()
    group = None

    def run(n):
        eb.init_canvas(canvas, committed, stop)
        for s in range(n):
            eb.step_split(sl[s % N], s % N, canvas, committed, H, amax, stop, group=group)

    run(W)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    full_t, rem = divmod(K, N)

    def region():
        for _ in range(full_t):
            run(N)
        if rem:
            run(rem)

    times = timed_regions(region, 3, barrier, stream)
    el = statistics.median(times)
    if dist is not None:
        t = torch.tensor([el], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        el = float(t.item())
    positions = K * w.L * w.B
    if rank == 0:
        line = {
            "metric": METRIC, "value": positions / (el * 1e-3), "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": el / K, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "canvas 1x256x262144 bf16, vocabulary split over the ranks",
                       "slice_width": hi - lo, "collective": "all_gather_into_tensor (NCCL)",
                       "timing": "eager steps (slice pass, all-gather, combine), median of 3 "
                                 "regions of exactly K steps"},
            "gpu_launches": K * 2 + (full_t + (1 if rem else 0)),
        }
        print(json.dumps(line), flush=True)
    eb.close()
    if dist is not None:
        dist.destroy_process_group()


def run_profile_case():
    """Three eager steps of the benchmark workload (about 0.4 GB on the device)."""
    import torch

    import entropy_bound_canvas_b200 as E
    import synth
    w = synth.WORKLOADS[WORKLOAD]
    dev = torch.device("cuda", 0)
    logits = [torch.empty((w.B, w.L, w.V), dtype=torch.bfloat16, device=dev) for _ in range(3)]
    for s in range(3):
        synth.generate_device(w, s, logits[s])
    eb = E.EBSampler(w.B, w.L, w.V, device=dev, **w.sampler_config())
    canvas, committed, stop = eb.new_canvas()
    H, amax = eb.outputs()
    for s in range(3):
        eb.step(logits[s], s, canvas, committed, H, amax, stop)
    torch.cuda.synchronize()
    assert eb.status() == 0
    eb.close()
    print("profile case done")


def run_profile_lmhead_case():
    """Three LM-head steps of a small case (1 x 256 positions, V = 32768,
    d = 2560; about 0.2 GB on the device)."""
    import torch

    import entropy_bound_canvas_b200 as E
    import synth
    from synth import lmhead as LM
    dev = torch.device("cuda", 0)
    w = synth.WORKLOADS["canvas"].replace(V=32768, seed=31)
    wc = LM.weight_codes(w.V, LMHEAD_D, seed=w.seed)
    W = LM.to_bf16(wc).to(dev)
    eb = E.EBSampler(w.B, w.L, w.V, device=dev, **w.sampler_config())
    canvas, committed, stop = eb.new_canvas()
    H, amax = eb.outputs()
    eb.init_canvas(canvas, committed, stop)
    for s in range(3):
        h = LM.to_bf16(LM.hidden_codes(wc, w.B, w.L, s, w.num_steps, seed=w.seed)).to(dev)
        eb.lmhead_step(h, W, s, canvas, committed, H, amax, stop)
    torch.cuda.synchronize()
    assert eb.status() == 0
    eb.close()
    print("lmhead profile case done")


def main():
    args = parse()
    if args.profile:
        run_profile_case()
        return
    if args.profile_lmhead:
        run_profile_lmhead_case()
        return
    if args.impl == "reference":
        run_reference(args)
    elif args.split_v:
        run_split_v(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
