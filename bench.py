"""Benchmark: the fused MoE layer megakernel (router -> top-k -> grouping ->
two grouped GEMMs -> weighted combine, one launch) on a Qwen3-30B-A3B-shaped
layer: hidden 2048, 128 experts, top-8, SwiGLU 768, Zipf(s) expert bias.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--T 128] [--sched dynamic]
                    [--zipf 1.2] [--impl reference]

One step = one MoE layer forward over T tokens.  Prints ONE JSON line on
rank 0.  `value` is the achieved algorithmic HBM bandwidth (GB/s) of the
whole job: the bytes the layer must move (the weights of every expert that
received a token, the router weights, X and Y) summed over ranks, divided by
the device time of a step (CUDA events on the launch stream, max over
ranks).  The L2 is flushed before every step, outside the timed events.
Several GPUs run independent replicas (the layer does not shard here).

The line also carries a timed `sweep` (T in {1, 16, 128, 1024, 4096}
x static / dynamic / hybrid / unfused schedules, Zipf 1.2, same binary) and
the CPU oracle timed on this host's cores (`cpu_baseline`: the whole layer,
single thread and all threads, median of 3).

--impl reference times the CPU oracle (plain C, fp64, all host threads) on
the whole layer, one layer per step, and prints the same line with
"impl": "reference".
"""
import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "fused MoE-layer latency µs & achieved HBM GB/s vs ~8 TB/s at T=1..4096 tokens"
EXPERT_BYTES = 2 * (2 * 768 * 2048 + 2048 * 768)  # W1 + W2 of one expert, bf16
WR_BYTES = 128 * 2048 * 2


def algorithmic_bytes(topk, T, hidden=2048):
    """Bytes the layer must move: weights of every expert that got a token,
    the router weights, X in, Y out, plus the small routing outputs."""
    touched = len(np.unique(np.asarray(topk)))
    return touched * EXPERT_BYTES + WR_BYTES + 2 * T * hidden * 2 + T * 8 * (4 + 4 + 4 + 4), touched


def moe_flops(T, hidden=2048, inter=768, E=128, k=8):
    return 2 * T * (E * hidden + k * (2 * inter * hidden + hidden * inter))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d.get("bf16_tflops"), "measured"
    return 6650.0, 1590.0, "fallback"


def load_traffic(T, sched):
    """dram read+write bytes per launch of the MoE kernel from the committed
    ncu summary, or None."""
    p = os.path.join(ROOT, "profiles", "moe_kernel_traffic.txt")
    if not os.path.exists(p):
        return None
    for line in open(p):
        f = line.split()
        if len(f) >= 4 and f[0] == "traffic" and f[1] == "T=%d" % T and f[2] == "sched=%s" % sched:
            return float(f[3].split("=")[1])
    return None


class ClockSampler:
    """SM clock and throttle reasons sampled through NVML while the timed
    region runs (reading only; no setting is changed)."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index):
        self.index = index
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None
            return self
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
            time.sleep(0.002)

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        names = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------------ GPU arm --
def combine_ranks(ms, e2e_ms, nbytes, world, device):
    """Whole-job figures of a replicas run: the max over ranks of the step
    times (device-timed) and the algorithmic bytes summed over ranks.  Every
    rank calls it (two all-reduces, in the same order on every rank)."""
    if world <= 1:
        return float(ms), float(e2e_ms), float(nbytes)
    import torch
    vals = torch.tensor([ms, e2e_ms, float(nbytes)], dtype=torch.float64, device=device)
    mx = vals.clone()
    torch.distributed.all_reduce(mx, op=torch.distributed.ReduceOp.MAX)
    sm = vals.clone()
    torch.distributed.all_reduce(sm, op=torch.distributed.ReduceOp.SUM)
    return float(mx[0]), float(mx[1]), float(sm[2])


def gpu_arm(args, rank, world, local_rank):
    import torch
    import event_driven_persistent_b200 as et

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    T, H, E, k = args.T, 2048, 128, 8
    d = _layer_inputs(T, args.zipf)

    def to_dev(a):
        a = np.ascontiguousarray(a)
        return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).to(dev)

    t = {n: to_dev(d[n]) for n in ("X", "Wr", "bias", "W1", "W2")}
    Y = torch.empty((T, H), dtype=torch.int16, device=dev)
    topk = torch.empty((T, k), dtype=torch.int32, device=dev)
    g = et.et_build_graph(et.ET_GRAPH_MOE, args.sched, max(T, args.max_T), device=local_rank)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)  # > 126 MB L2

    def step(with_topk=False):
        et.et_run_moe(g, T, t["X"], t["Wr"], t["bias"], t["W1"], t["W2"], Y, topk if with_topk else None,
                      stream=stream)

    step(True)
    if et.et_sync_status(g, stream) != 0:
        raise RuntimeError("MoE run reported a device error")
    nbytes, touched = algorithmic_bytes(topk.cpu().numpy(), T)

    clk = ClockSampler(local_rank).__enter__()  # sampled over the timed region, the sweep and e2e
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.zero_()
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    st = et.et_sync_status(g, stream)
    if st != 0:
        raise RuntimeError("MoE run reported a device error: %s" % et.et_status_str(st))
    times = [a.elapsed_time(b) for a, b in evs]  # ms
    ms = statistics.median(times)
    sweep = run_sweep(args, et, g, t, dev, stream, flush) if (args.sweep and world == 1) else None

    # end to end through the C ABI with host buffers: H2D of X, the layer, D2H of Y
    Xh = torch.from_numpy(np.ascontiguousarray(d["X"]).view(np.int16)).pin_memory()
    Yh = torch.empty((T, H), dtype=torch.int16).pin_memory()
    Xd = torch.empty_like(t["X"])
    e2e_ms = []
    for i in range(args.warmup + args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        Xd.copy_(Xh, non_blocking=True)
        et.et_run_moe(g, T, Xd, t["Wr"], t["bias"], t["W1"], t["W2"], Y, stream=stream)
        Yh.copy_(Y, non_blocking=True)
        b.record(stream)
        b.synchronize()
        if i >= args.warmup:
            e2e_ms.append(a.elapsed_time(b))
    e2e = statistics.median(e2e_ms)
    clk.__exit__()

    ms, e2e, tot_bytes = combine_ranks(ms, e2e, nbytes, world, dev)
    et.et_destroy_graph(g)
    if rank != 0:
        return None
    hbm, tc, src = load_peaks()
    achieved = nbytes / (ms * 1e-3) / 1e9
    flops = moe_flops(T)
    return {
        "metric": METRIC, "value": round(tot_bytes / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
        "latency_us": round(ms * 1e3, 2), "latency_us_p10_p90": [round(float(np.percentile(times, 10)) * 1e3, 2),
                                                                 round(float(np.percentile(times, 90)) * 1e3, 2)],
        "latency_us_mean": round(float(np.mean(times)) * 1e3, 2), "timing": "median of the timed steps",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "MoE layer T=%d, hidden 2048, 128 experts top-8, SwiGLU 768, Zipf s=%g bias, "
                               "%s schedule" % (T, args.zipf, args.sched),
                   "T": T, "sched": args.sched, "zipf_s": args.zipf, "experts_touched": touched,
                   "l2": "flushed (256 MB write) before every step, outside the timed events",
                   "parallelism": "replicas" if world > 1 else "single"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                     "frac": round(achieved / hbm, 4), "peak_source": src + " (MEASURED_PEAKS.json hbm_gbs)",
                     "traffic": load_traffic(T, args.sched), "bytes_per_launch": nbytes,
                     "tensor_frac": round(flops / (ms * 1e-3) / (tc * 1e12), 4) if tc else None},
        "e2e": {"value": round(tot_bytes / (e2e * 1e-3) / 1e9, 2), "unit": "GB/s", "latency_us": round(e2e * 1e3, 2),
                "h2d_bytes_per_step": int(Xh.numel() * 2), "d2h_bytes_per_step": int(Yh.numel() * 2)},
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
        "sweep": sweep,
    }


def run_sweep(args, et, g_dyn, t, dev, stream, flush):
    """Device time of the layer over the token range and the four schedules
    (same binary; one graph per schedule, max_T 4096), Zipf s = 1.2: median
    of `sweep_steps` launches, L2 flushed before each."""
    import torch
    hbm, tc, _ = load_peaks()
    graphs = {"dynamic": g_dyn}
    for s in ("static", "hybrid", "unfused"):
        graphs[s] = et.et_build_graph(et.ET_GRAPH_MOE, s, max(4096, args.max_T), device=dev.index)
    out = []
    try:
        for T in (1, 16, 128, 1024, 4096):
            x = W.moe_inputs(T, weights=False)["X"]   # the weights and bias are the benchmark's own
            X = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(dev)
            Y = torch.empty((T, 2048), dtype=torch.int16, device=dev)
            topk = torch.empty((T, 8), dtype=torch.int32, device=dev)
            row = {"T": T}
            for s, g in graphs.items():
                et.et_run_moe(g, T, X, t["Wr"], t["bias"], t["W1"], t["W2"], Y, topk, stream=stream)
                if et.et_sync_status(g, stream) != 0:
                    raise RuntimeError("sweep run reported a device error")
                nbytes, touched = algorithmic_bytes(topk.cpu().numpy(), T)
                ts = []
                for i in range(3 + args.sweep_steps):
                    flush.zero_()
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record(stream)
                    et.et_run_moe(g, T, X, t["Wr"], t["bias"], t["W1"], t["W2"], Y, stream=stream)
                    b.record(stream)
                    b.synchronize()
                    if i >= 3:
                        ts.append(a.elapsed_time(b))
                if et.et_sync_status(g, stream) != 0:
                    raise RuntimeError("sweep run reported a device error")
                ms = statistics.median(ts)
                row[s] = {"us": round(ms * 1e3, 2), "GB/s": round(nbytes / (ms * 1e-3) / 1e9, 1),
                          "hbm_frac": round(nbytes / (ms * 1e-3) / 1e9 / hbm, 4),
                          "tensor_frac": round(moe_flops(T) / (ms * 1e-3) / (tc * 1e12), 4) if tc else None}
                row["experts_touched"] = touched
            out.append(row)
    finally:
        for s in ("static", "hybrid", "unfused"):
            et.et_destroy_graph(graphs[s])
    return {"zipf_s": args.zipf, "steps_per_point": args.sweep_steps, "timing": "median, L2 flushed before each launch",
            "points": out}


# ------------------------------------------- other workloads (one GPU) --
MLP_BYTES = 2 * (2 * 14336 * 4096 + 4096 * 14336)  # Wgu + Wd, bf16


def other_arm(args):
    """--workload mlp (decode MLP, static schedule, batch --B) or splitk
    (2048 x 128 fp32, static): device time of one megakernel launch with
    the L2 flushed before it, and the achieved algorithmic HBM GB/s."""
    import torch
    import event_driven_persistent_b200 as et
    dev = torch.device("cuda", 0)

    def to_dev(a):
        a = np.ascontiguousarray(a)
        return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).to(dev)

    control = None  # (description, callable) of a control timed beside the workload
    if args.workload == "decode":
        B = args.B
        d = W.decode_inputs(B)
        wkeys = ("g1", "Wqkv", "gq", "gk", "Wo", "g2", "Wgu", "Wd")
        d["Vc"] = W.v_cache_device(d["Vc"])  # the device's V cache layout
        t = {n: to_dev(d[n]) for n in wkeys + ("X", "pos", "Kc", "Vc")}
        Y = torch.empty((B, 4096), dtype=torch.int16, device=dev)
        sched = args.sched
        g = et.et_build_graph(et.ET_GRAPH_DECODE, sched, 64)
        run = lambda: et.et_run_decode(g, B, t["X"], t["pos"], t, t["Kc"], t["Vc"], Y)  # noqa: E731
        wbytes = sum(d[n].nbytes for n in wkeys)
        kv = int(np.sum(d["pos"].astype(np.int64) + 1)) * 8 * 128 * 2 * 2   # K and V read, new entry included
        nbytes = wbytes + kv + B * 8 * 128 * 2 * 2 + 2 * B * 4096 * 2     # + appended K, V; X in, Y out
        workload = ("Llama-3-8B-shaped decode layer B=%d (hidden 4096, 32/8 heads x 128, SwiGLU 14336, "
                    "context %d..%d, mean %.0f), %s schedule" % (B, d["pos"].min(), d["pos"].max(),
                                                                 d["pos"].mean(), sched))
    elif args.workload == "moe_mlp":
        T = args.T if args.T <= 128 else 128
        d = W.moe_inputs(T, zipf_s=args.zipf)
        m = W.dense_mlp_weights()
        t = {n: to_dev(v) for n, v in list(d.items()) + list(m.items())}
        Y1 = torch.empty((T, 2048), dtype=torch.int16, device=dev)
        Y2 = torch.empty((T, 2048), dtype=torch.int16, device=dev)
        topk = torch.empty((T, 8), dtype=torch.int32, device=dev)
        sched = args.sched
        g = et.et_build_graph(et.ET_GRAPH_MOE_MLP, sched, 128)
        g_moe = et.et_build_graph(et.ET_GRAPH_MOE, sched, 128)
        g_mlp = et.et_build_graph(et.ET_GRAPH_MLP, "static" if sched == "dynamic" else sched, 128, hidden=2048,
                                  inter=6144)
        et.et_run_moe(g_moe, T, t["X"], t["Wr"], t["bias"], t["W1"], t["W2"], Y1, topk)
        if et.et_sync_status(g_moe) != 0:
            raise RuntimeError("MoE run reported a device error")
        nbytes = algorithmic_bytes(topk.cpu().numpy(), T)[0] + sum(m[n].nbytes for n in ("gamma", "Wgu", "Wd")) + \
            2 * T * 2048 * 2

        def two():
            et.et_run_moe(g_moe, T, t["X"], t["Wr"], t["bias"], t["W1"], t["W2"], Y1)
            et.et_run_mlp(g_mlp, T, Y1, t["gamma"], t["Wgu"], t["Wd"], Y2)

        run = lambda: et.et_run_moe_mlp(g, T, t["X"], t["Wr"], t["bias"], t["W1"], t["W2"], t["gamma"],  # noqa: E731
                                        t["Wgu"], t["Wd"], Y1, Y2)
        control = ("two launches (MoE megakernel, then the dense-MLP megakernel)", two)
        workload = ("MoE layer T=%d (Zipf %g) -> dense MLP 2048->6144->2048, one megakernel, %s schedule"
                    % (T, args.zipf, sched))
    elif args.workload == "mlp":
        B = args.B
        d = W.mlp_inputs(B)
        t = {n: to_dev(d[n]) for n in ("X", "gamma", "Wgu", "Wd")}
        Y = torch.empty((B, 4096), dtype=torch.int16, device=dev)
        g = et.et_build_graph(et.ET_GRAPH_MLP, args.sched, 64)
        run = lambda: et.et_run_mlp(g, B, t["X"], t["gamma"], t["Wgu"], t["Wd"], Y)
        nbytes = MLP_BYTES + 8192 + 16384 * B
        workload = "decode MLP B=%d, hidden 4096, SwiGLU 14336, %s schedule" % (B, args.sched)
    else:
        A = to_dev(W.splitk_inputs(2048))
        Bp = torch.zeros((2048, 4), device=dev)
        C = torch.zeros((2048,), device=dev)
        g = et.et_build_graph(et.ET_GRAPH_SPLITK, args.sched, 2048)
        run = lambda: et.et_run_splitk(g, A, 2048, Bp, C)  # noqa: E731
        control = ("two launches (partials kernel, then finals kernel)",
                   lambda: et.et_run_splitk_two_launch(A, 2048, 128, 32, Bp, C))
        nbytes = 2048 * 128 * 4 + 2048 * 5 * 4
        workload = "split-K 2048 x 128 fp32, chunks of 32, %s schedule" % args.sched
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def timed(fn):
        for _ in range(args.warmup):
            flush.zero_()
            fn()
        torch.cuda.synchronize(dev)
        ts = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    ms = timed(run)
    if et.et_sync_status(g) != 0:
        raise RuntimeError("run reported a device error")
    extra = {}
    if control is not None:
        ms_c = timed(control[1])
        extra["control"] = {"what": control[0], "latency_us": round(ms_c * 1e3, 2)}
    et.et_destroy_graph(g)
    hbm, _, src = load_peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": workload, "latency_us": round(ms * 1e3, 2), "value": round(gbs, 1), "unit": "GB/s",
            "steps": args.steps, "warmup": args.warmup, "bytes_per_launch": nbytes, **extra,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(gbs / hbm, 4), "peak_source": src}}


# ------------------------------------------------------------ CPU oracle --
_INPUTS = {}


def _layer_inputs(T, zipf):
    """The seeded layer inputs, generated once per process (generation is
    not part of any timed region)."""
    if (T, zipf) not in _INPUTS:
        _INPUTS[(T, zipf)] = W.moe_inputs(T, zipf_s=zipf)
    return _INPUTS[(T, zipf)]


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def oracle_layer_seconds(T, zipf, threads):
    """One whole MoE layer through the oracle (router logits, top-8 +
    softmax, grouping, both grouped GEMMs per routed pair, combine) on
    `threads` host threads; returns (seconds, algorithmic bytes)."""
    import oracle
    d = _layer_inputs(T, zipf)
    oracle.set_threads(threads)
    t0 = time.perf_counter()
    out = oracle.moe(d["X"], d["Wr"], d["bias"], d["W1"], d["W2"], 8)
    el = time.perf_counter() - t0
    nbytes, _ = algorithmic_bytes(out["topk"], T)
    return el, nbytes


def cpu_oracle(args, reps=3):
    """The oracle as it stands, timed on this host: the whole layer at the
    benchmark's T, median of `reps` runs on one thread and on every thread."""
    import oracle
    n_all = oracle.max_threads()
    res = {}
    for threads in (1, n_all):
        ts = []
        for _ in range(reps):
            el, nbytes = oracle_layer_seconds(args.T, args.zipf, threads)
            ts.append(el)
        res[threads] = (statistics.median(ts), nbytes)
    (s_all, nbytes), (s_one, _) = res[n_all], res[1]
    return {"value": round(nbytes / s_all / 1e9, 4), "unit": "GB/s", "cores": n_all, "kind": "oracle",
            "sample": "whole layer T=%d (router, top-8, grouping, both grouped GEMMs, combine), median of %d runs "
                      "on %d threads (OpenMP over tokens / routed pairs)" % (args.T, reps, n_all),
            "latency_us": round(s_all * 1e6, 1), "nproc": os.cpu_count(), "cpu_model": cpu_model(),
            "single_thread": {"value": round(nbytes / s_one / 1e9, 4), "latency_us": round(s_one * 1e6, 1),
                              "cores": 1, "sample": "same layer, median of %d runs on one thread" % reps}}


def reference_arm(args, budget_s=180.0):
    """The oracle as it stands on this host's threads, one whole layer per
    step.  Steps beyond what fits in `budget_s` (after the first timed step)
    are not run; `steps` reports how many were."""
    import oracle
    n_all = oracle.max_threads()
    for _ in range(args.warmup):
        oracle_layer_seconds(args.T, args.zipf, n_all)
    ts, nbytes = [], 0
    t_start = time.perf_counter()
    for i in range(args.steps):
        el, nbytes = oracle_layer_seconds(args.T, args.zipf, n_all)
        ts.append(el)
        if time.perf_counter() - t_start + el > budget_s:
            break
    sec = statistics.median(ts)
    v = round(nbytes / sec / 1e9, 4)
    sample = ("whole layer T=%d per step (router, top-8, grouping, both grouped GEMMs, combine) on %d threads; "
              "%d of %d requested steps run within %.0f s" % (args.T, n_all, len(ts), args.steps, budget_s))
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "latency_us": round(sec * 1e6, 1),
            "n_gpus": args.gpus, "steps": len(ts), "steps_requested": args.steps, "warmup": args.warmup,
            "ms_per_step": round(sec * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "MoE layer T=%d, hidden 2048, 128 experts top-8, SwiGLU 768, Zipf s=%g bias, "
                                   "%s schedule" % (args.T, args.zipf, args.sched),
                       "T": args.T, "sched": args.sched, "zipf_s": args.zipf},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": n_all, "kind": "oracle", "sample": sample,
                             "nproc": os.cpu_count(), "cpu_model": cpu_model()},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--T", type=int, default=128)
    ap.add_argument("--max_T", type=int, default=4096)
    ap.add_argument("--sched", default="dynamic", choices=["static", "dynamic", "unfused", "hybrid"])
    ap.add_argument("--zipf", type=float, default=1.2)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default="moe", choices=["moe", "mlp", "splitk", "decode", "moe_mlp"],
                    help="moe (the benchmark line); mlp, splitk, decode or moe_mlp print a kernel timing line")
    ap.add_argument("--B", type=int, default=1, help="batch (--workload mlp or decode)")
    ap.add_argument("--no-sweep", dest="sweep", action="store_false", help="skip the T x schedule sweep")
    ap.add_argument("--sweep-steps", type=int, default=50)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))

    if args.workload != "moe":
        if args.sched == "dynamic" and "--sched" not in sys.argv:
            args.sched = "static"
        print(json.dumps(other_arm(args)))
        return

    if args.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(reference_arm(args)))
        return

    if world > 1:
        import datetime
        import torch
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    line = gpu_arm(args, rank, world, local_rank)
    if world > 1:
        import torch
        torch.distributed.destroy_process_group()
    if rank == 0:
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_oracle(args)
        print(json.dumps(line))


if __name__ == "__main__":
    main()
