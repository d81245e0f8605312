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

--impl reference times the CPU oracle (plain C, fp64) on this host, on a
bounded sample of the same workload, and prints the same line with
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

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(local_rank) as clk:
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
    ms = sum(times) / len(times)

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
    e2e = sum(e2e_ms) / len(e2e_ms)

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
    }


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

    if args.workload == "mlp":
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
        run = lambda: et.et_run_splitk(g, A, 2048, Bp, C)
        nbytes = 2048 * 128 * 4 + 2048 * 5 * 4
        workload = "split-K 2048 x 128 fp32, chunks of 32, %s schedule" % args.sched
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        flush.zero_()
        run()
    torch.cuda.synchronize(dev)
    times = []
    for _ in range(args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        run()
        b.record()
        b.synchronize()
        times.append(a.elapsed_time(b))
    if et.et_sync_status(g) != 0:
        raise RuntimeError("run reported a device error")
    et.et_destroy_graph(g)
    ms = sum(times) / len(times)
    hbm, _, src = load_peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": workload, "latency_us": round(ms * 1e3, 2), "value": round(gbs, 1), "unit": "GB/s",
            "steps": args.steps, "warmup": args.warmup, "bytes_per_launch": nbytes,
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


def cpu_oracle(args, budget_s=15.0):
    """The oracle as it stands (single thread) on a bounded token sample of
    the same layer: per-token evaluation (router, top-8, eight experts,
    combine).  The layer time is the per-token time x T."""
    import oracle
    T = args.T
    d = _layer_inputs(T, args.zipf)
    ntok, el = 0, 0.0
    t0 = time.perf_counter()
    while ntok < T and time.perf_counter() - t0 < budget_s:
        oracle.moe_per_token(d["X"], d["Wr"], d["bias"], d["W1"], d["W2"], [ntok], 8)
        ntok += 1
    el = time.perf_counter() - t0
    logits = oracle.router_logits(d["X"], d["Wr"], d["bias"])
    tk, _ = oracle.topk_softmax(logits, 8)
    nbytes, _ = algorithmic_bytes(tk, T)
    layer_s = el / ntok * T
    return {"value": round(nbytes / layer_s / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": "%d of %d tokens evaluated per token (router, top-8, 8 experts, combine) in %.1f s; "
                      "layer time = per-token time x T" % (ntok, T, el),
            "latency_us": round(layer_s * 1e6, 1)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--T", type=int, default=128)
    ap.add_argument("--max_T", type=int, default=4096)
    ap.add_argument("--sched", default="dynamic", choices=["static", "dynamic", "unfused"])
    ap.add_argument("--zipf", type=float, default=1.2)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default="moe", choices=["moe", "mlp", "splitk"],
                    help="moe (the benchmark line); mlp or splitk print a kernel timing line")
    ap.add_argument("--B", type=int, default=1, help="decode MLP batch (--workload mlp)")
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
        times = []
        for i in range(args.warmup + args.steps):
            r = cpu_oracle(args, budget_s=max(2.0, 60.0 / (args.warmup + args.steps)))
            if i >= args.warmup:
                times.append(r)
        v = statistics.median(x["value"] for x in times)
        lat = statistics.median(x["latency_us"] for x in times)
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "latency_us": lat,
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(lat / 1e3, 3), "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": "MoE layer T=%d, hidden 2048, 128 experts top-8, SwiGLU 768, Zipf s=%g bias"
                                       % (args.T, args.zipf), "T": args.T, "zipf_s": args.zipf},
                "cpu_baseline": {"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle",
                                 "sample": times[-1]["sample"]},
                "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
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
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_oracle(args)
        print(json.dumps(line))


if __name__ == "__main__":
    main()
