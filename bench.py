"""Throughput benchmark of the FP4 microscaling hot path on B200.

Default workload (N = 1): the block-size x scale-format sweep on five bf16 4096x4096 tensors
N(0, sigma^2), sigma in {0.005, 0.01, 0.02, 0.05, 0.1}; block sizes {4..256} x {E4M3, UE5M3} = 70
points.  One step = the fused pass (quantize + pack + three-term error reduction, x read once) of
every point, then dequantize (bf16 out) of every point; sigma innermost, so that no buffer is
re-read while it could still sit in L2 (inputs 168 MB > 126 MB L2, outputs ~1.8 GB per step).
The device-resident number replays one CUDA graph per phase; `e2e` calls the public Python API
eagerly, every step copying its five inputs from pinned host memory and its 70 error records back
(two sets of device buffers: step i + 1's input copies overlap step i's kernels).
The plain quantize + pack kernel (no error reduction) is timed beside the step the same way.

Byte accounting (algorithmic, bf16): fused pass and quantize 2 + 1/2 + 1/N bytes per element,
dequantize 1/2 + 1/N + 2.  `roofline` covers the fused pass, the dominant kernel of the step.

--gpus N > 1 runs under torchrun, one process per GPU: every rank runs the same sweep on its own
seeded tensors (weak scaling; the path has no exchange step), timing is the max over ranks.
--impl reference times the CPU oracle on a bounded sample of the same workload.
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantize+pack / dequant GB/s and Gelem/s on 1 B200; fraction of HBM peak"
WORKLOAD = "bf16-4096x4096 x5 sigma sweep, blocks 4..256 x {E4M3,UE5M3} (70 points)"
SHAPE = (4096, 4096)
L2_BYTES = 126 * 2 ** 20
# DRAM bytes (read + write) of one grouped fused-pass launch (5 tensors, N = 32, E4M3), from the
# ncu capture summarised in profiles/k_error_stats_bf16_fused_group5_4096x4096_n32.md: every x is
# read once, most of the codes and scales are still in L2 when the launch ends.
FUSED_TRAFFIC_BYTES = 167834368 + 8116736


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    # single-kernel timing / profiling case (not the benchmark line)
    ap.add_argument("--case", choices=["quantize", "dequantize", "stats", "stats-recompute",
                                       "quantize-stats", "global-scale", "fake-quantize",
                                       "matmul"])
    ap.add_argument("--mnk", type=int, nargs=3, default=[8192, 8192, 8192],
                    help="m n k of --case matmul")
    ap.add_argument("--shape", type=int, nargs=2, default=[16384, 8192])
    ap.add_argument("--block", type=int, default=32)
    ap.add_argument("--fmt", choices=["e4m3", "ue5m3"], default="e4m3")
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--group", type=int, default=1, help="tensors per grouped launch (--case)")
    ap.add_argument("--rotate", type=int, default=1,
                    help="--case: cycle R independent input sets, 4R launches between two events "
                         "(no flush: each set is evicted by the others), instead of one flushed "
                         "launch per event pair")
    return ap.parse_args(argv)


def points():
    from fp4_microscaling_tensor_b200 import inputs
    pts = []
    for n in inputs.SWEEP_BLOCKS:
        for fmt in (0, 1):
            for k in range(len(inputs.SWEEP_SIGMAS)):  # sigma innermost
                pts.append((k, n, fmt))
    return pts


def q_bytes(numel, n):
    return numel * (2 + 0.5 + 1.0 / n)


def step_bytes(pts, numel):
    q = sum(q_bytes(numel, n) for _, n, _ in pts)
    return q, q  # fused quantize + pack + error reduction, dequantize


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """SM clock, power and throttle reasons sampled every 5 ms (NVML) while the timed region runs.

    Sampling starts before and stops after the region.  Falls back to `nvidia-smi -lms 200`."""

    def __init__(self, device):
        import threading
        self.device = device
        self.samples = []
        self.stop = threading.Event()
        self.thread = None
        self.nvml = None
        self.handle = None
        self.smi = None

    def _open_nvml(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.device).uuid)
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(
                uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(self.device.index or 0)
        self.nvml = pynvml

    def _loop(self):
        nv, h = self.nvml, self.handle
        reasons = {"hw_slowdown": nv.nvmlClocksThrottleReasonHwSlowdown,
                   "hw_thermal_slowdown": nv.nvmlClocksThrottleReasonHwThermalSlowdown,
                   "sw_thermal_slowdown": nv.nvmlClocksThrottleReasonSwThermalSlowdown,
                   "sw_power_cap": nv.nvmlClocksThrottleReasonSwPowerCap}
        while not self.stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                mask = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                util = nv.nvmlDeviceGetUtilizationRates(h).gpu
                self.samples.append((sm, [k for k, b in reasons.items() if mask & b], pw, util))
            except Exception:
                pass
            self.stop.wait(0.005)

    def __enter__(self):
        import threading
        try:
            self._open_nvml()
            self.thread = threading.Thread(target=self._loop, daemon=True)
            self.thread.start()
        except Exception:
            self.nvml = None
            try:
                self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
                self.smi = subprocess.Popen(
                    ["nvidia-smi", "--query-gpu=clocks.sm,clocks_event_reasons.active",
                     "--format=csv,noheader,nounits", "-lms", "200"],
                    stdout=self.tmp, stderr=subprocess.DEVNULL)
            except FileNotFoundError:
                self.smi = None
        time.sleep(0.05)
        return self

    def __exit__(self, *a):
        time.sleep(0.02)
        self.stop.set()
        if self.thread is not None:
            self.thread.join(timeout=2)
        if self.smi is not None:
            self.smi.terminate()
            self.smi.wait(timeout=5)

    def summary(self):
        max_mhz = None
        if self.nvml is not None:
            try:
                max_mhz = self.nvml.nvmlDeviceGetMaxClockInfo(self.handle, self.nvml.NVML_CLOCK_SM)
            except Exception:
                pass
        if self.samples:
            sm = [s[0] for s in self.samples]
            busy = [s[0] for s in self.samples if s[3] > 0] or sm
            reasons = sorted({r for s in self.samples for r in s[1]})
            return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max_mhz, "reasons": reasons,
                    "samples": len(self.samples), "power_w_max": max(s[2] for s in self.samples),
                    "source": "nvml 5 ms"}
        if self.smi is not None:
            rows = []
            with open(self.tmp.name) as f:
                for line in f:
                    p = [c.strip() for c in line.split(",")]
                    if p and p[0].isdigit():
                        rows.append(int(p[0]))
            os.unlink(self.tmp.name)
            if rows:
                return {"sm_mhz": statistics.median(rows), "sm_max_mhz": max_mhz, "reasons": [],
                        "samples": len(rows), "source": "nvidia-smi 200 ms"}
        return {"sm_mhz": None, "sm_max_mhz": max_mhz, "reasons": ["no clock samples"]}


# ------------------------------------------------------------------------------------------------
# CPU oracle: baseline leg and the reference arm
# ------------------------------------------------------------------------------------------------

def oracle_sample_step(xs_host, rows, pts, threads):
    """Quantize, error-reduce and dequantize the first `rows` rows of every point on the CPU."""
    import oracle
    cols = SHAPE[1]
    for k, n, fmt in pts:
        x = xs_host[k][: rows * cols]
        p, s = oracle.quantize(x, rows, cols, n, fmt, threads=threads)
        oracle.dequantize(p, s, rows, cols, n, fmt, out_bf16=True, threads=threads)
        oracle.error_stats(x, rows, cols, n, fmt, packed=p, scales=s, threads=threads)


def oracle_sample(seconds, threads):
    """Pick a row count whose oracle step takes about `seconds`; return (xs_host, rows, pts)."""
    from fp4_microscaling_tensor_b200 import inputs
    pts = points()
    xs = [inputs.to_oracle(inputs.workload2(k, shape=SHAPE)) for k in range(5)]
    oracle_sample_step(xs, 4, pts, threads)  # warm-up (thread pool, caches)
    t0 = time.perf_counter()
    oracle_sample_step(xs, 32, pts, threads)
    per_row = (time.perf_counter() - t0) / 32
    rows = int(max(1, min(SHAPE[0], seconds / max(per_row, 1e-9))))
    return xs, rows, pts


def cpu_rate(xs, rows, pts, threads, reps=1):
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle_sample_step(xs, rows, pts, threads)
    dt = (time.perf_counter() - t0) / reps
    numel = rows * SHAPE[1]
    qb, db = step_bytes(pts, numel)
    return (qb + db) / dt / 1e9, dt


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    threads = os.cpu_count() or 1
    xs, rows, pts = oracle_sample(args.cpu_seconds / 2, threads)
    for _ in range(args.warmup):
        oracle_sample_step(xs, rows, pts, threads)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_sample_step(xs, rows, pts, threads)
        times.append(time.perf_counter() - t0)
    dt = sum(times) / len(times)
    numel = rows * SHAPE[1]
    qb, db = step_bytes(pts, numel)
    v = (qb + db) / dt / 1e9
    sample = f"first {rows} of 4096 rows of each of the 70 points (quantize, error reduction, dequantize)"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": WORKLOAD, "sample_rows": rows},
        "cpu_baseline": {"value": v, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ------------------------------------------------------------------------------------------------
# GPU arm
# ------------------------------------------------------------------------------------------------

class Sweep:
    """Device buffers and the phases of one sweep step.  The five sigma tensors of one (N, format)
    point are one grouped launch (14 launches per phase)."""

    def __init__(self, xs, device):
        import torch
        import fp4_microscaling_tensor_b200 as mx
        self.mx = mx
        self.xs = xs
        self.pts = points()
        rows, cols = SHAPE
        self.packed = [torch.empty(rows, cols // 2, dtype=torch.uint8, device=device)
                       for _ in self.pts]
        self.scales = [torch.empty(rows, cols // n, dtype=torch.uint8, device=device)
                       for _, n, _ in self.pts]
        self.ys = [torch.empty(rows, cols, dtype=torch.bfloat16, device=device) for _ in self.pts]
        self.stats = torch.empty(len(self.pts), 64, dtype=torch.uint8, device=device)
        self.ws = mx.stats_workspace(device)
        # groups: consecutive points that share (N, format), i.e. the sigma tensors
        self.groups = []
        for i, (k, n, fmt) in enumerate(self.pts):
            if self.groups and self.groups[-1][1:] == (n, fmt):
                self.groups[-1][0].append(i)
            else:
                self.groups.append(([i], n, fmt))

    def phase_q(self):
        for idx, n, fmt in self.groups:
            self.mx.quantize_group([self.xs[self.pts[i][0]] for i in idx], n, fmt,
                                   packed=[self.packed[i] for i in idx],
                                   scales=[self.scales[i] for i in idx])

    def phase_qs(self):
        for idx, n, fmt in self.groups:
            self.mx.quantize_with_stats_group(
                [self.xs[self.pts[i][0]] for i in idx], n, fmt,
                packed=[self.packed[i] for i in idx], scales=[self.scales[i] for i in idx],
                out=self.stats[idx[0]:idx[-1] + 1], workspace=self.ws)

    def phase_dq(self):
        for idx, n, fmt in self.groups:
            self.mx.dequantize_group([self.packed[i] for i in idx], [self.scales[i] for i in idx],
                                     n, fmt, out=[self.ys[i] for i in idx])

    def step(self):
        self.phase_qs()
        self.phase_dq()


def time_graphs(graphs, steps, stream):
    """Replay the graphs `steps` times; per-graph device seconds summed over the steps."""
    import torch
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(graphs) + 1)]
          for _ in range(steps)]
    with torch.cuda.stream(stream):
        for s in range(steps):
            ev[s][0].record(stream)
            for j, g in enumerate(graphs):
                g.replay()
                ev[s][j + 1].record(stream)
    stream.synchronize()
    return [sum(ev[s][j].elapsed_time(ev[s][j + 1]) for s in range(steps)) / 1e3
            for j in range(len(graphs))]


def small_tensor_latency(dev, stream, calls=1000):
    """Microseconds per call for the fp32 256 x 256 tensor (N = 32, E4M3): quantize, dequantize
    (fp32 out), error reduction from the stored codes, each replayed as one graph of `calls`."""
    import torch
    import fp4_microscaling_tensor_b200 as mx
    from fp4_microscaling_tensor_b200 import inputs
    x = inputs.workload1(device=dev)
    p, s = mx.quantize(x, 32, mx.E4M3)
    y = torch.empty_like(x)
    out = torch.empty(64, dtype=torch.uint8, device=dev)
    ws = mx.stats_workspace(dev)
    fns = {"quantize": lambda: mx.quantize(x, 32, mx.E4M3, packed=p, scales=s),
           "dequantize": lambda: mx.dequantize(p, s, 32, mx.E4M3, out_dtype=torch.float32, out=y),
           "error_stats": lambda: mx.error_stats(x, 32, mx.E4M3, packed=p, scales=s, out=out,
                                                 workspace=ws)}
    res = {}
    for name, fn in fns.items():
        with torch.cuda.stream(stream):
            fn()
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(calls):
                fn()
        with torch.cuda.stream(stream):
            g.replay()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        stream.synchronize()
        res[name] = e0.elapsed_time(e1) * 1e3 / calls
        del g
    return res


def rank_seed(k, rank):
    """Seed of sigma index k on a rank: every rank draws its own tensors (weak scaling)."""
    return 100 + k + 1000 * rank


def max_over_ranks(vals, device):
    """Element-wise max over the ranks of the process group (identity on one process)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in vals]
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def run_ours(args):
    import torch
    import torch.distributed as dist

    import fp4_microscaling_tensor_b200 as mx
    from fp4_microscaling_tensor_b200 import inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)

    rows, cols = SHAPE
    numel = rows * cols
    # each rank draws its own tensors (seed offset by rank): weak scaling, no data exchange
    xs = []
    for k in range(len(inputs.SWEEP_SIGMAS)):
        x = inputs.normal(SHAPE, inputs.SWEEP_SIGMAS[k], rank_seed(k, rank), device=dev)
        xs.append(x)
    sw = Sweep(xs, dev)
    qb, db = step_bytes(sw.pts, numel)

    # eager warm-up (also loads every kernel), then one graph per phase
    with torch.cuda.stream(stream):
        sw.step()
        sw.phase_q()
    stream.synchronize()
    graphs = []
    n0 = mx.kernel_launches()
    for fn in (sw.phase_qs, sw.phase_dq):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        graphs.append(g)
    launches_per_step = mx.kernel_launches() - n0
    g_q = torch.cuda.CUDAGraph()  # plain quantize + pack, timed beside the step
    with torch.cuda.graph(g_q, stream=stream):
        sw.phase_q()

    def barrier():
        if world > 1:
            dist.barrier()

    time_graphs(graphs, args.warmup, stream)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        t_wall = time.perf_counter()
        ph = time_graphs(graphs, args.steps, stream)
        t_wall = time.perf_counter() - t_wall
    barrier()
    torch.cuda.synchronize()
    total = sum(ph)
    comb = max_over_ranks([total] + ph, dev)
    total, ph = comb[0], comb[1:]
    step_s = total / args.steps
    value = world * (qb + db) / step_s / 1e9

    # plain quantize + pack of the same 70 points (not part of the step)
    q_steps = max(3, min(args.steps, 50))
    time_graphs([g_q], 3, stream)
    t_q = max_over_ranks([time_graphs([g_q], q_steps, stream)[0] / q_steps], dev)[0]

    # ---- the small fp32 tensor (256 x 256, N = 32, E4M3): latency per call, one graph of 1000
    #      calls per kernel (launch-bound; reported beside the throughput, no roofline claim)
    small = small_tensor_latency(dev, stream)

    # ---- end to end through the public API: every step copies its five inputs from pinned host
    #      memory and its 70 error records back; two sets of device buffers let step i + 1's
    #      input copies (copy stream) run while step i computes (compute stream)
    host = [x.cpu().pin_memory() for x in xs]
    copy_stream = torch.cuda.Stream(device=dev)
    bufs = []
    for _ in range(2):
        dxs = [torch.empty_like(x) for x in xs]
        bufs.append({"xs": dxs, "sw": Sweep(dxs, dev),
                     "stats": torch.empty(len(sw.pts), 64, dtype=torch.uint8).pin_memory(),
                     "ready": torch.cuda.Event(), "free": torch.cuda.Event()})

    def e2e_steps(n):
        for i in range(n):
            b = bufs[i % 2]
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(b["free"])      # step i - 2 is done with these inputs
                for h, d in zip(host, b["xs"]):
                    d.copy_(h, non_blocking=True)
                b["ready"].record(copy_stream)
            with torch.cuda.stream(stream):
                stream.wait_event(b["ready"])
                b["sw"].step()
                b["stats"].copy_(b["sw"].stats, non_blocking=True)
                b["free"].record(stream)
        stream.synchronize()
        copy_stream.synchronize()

    e2e_steps(2)
    barrier()
    t0 = time.perf_counter()
    e2e_steps(args.e2e_steps)
    e2e_s = max_over_ranks([(time.perf_counter() - t0) / args.e2e_steps], dev)[0]
    h2d = sum(x.numel() * x.element_size() for x in xs)
    d2h = bufs[0]["stats"].numel()

    # ---- a second replay of the fused phase gives the same error records (deterministic sums)
    stats_a = sw.stats.clone()
    with torch.cuda.stream(stream):
        graphs[0].replay()
    stream.synchronize()
    deterministic = bool(torch.equal(stats_a, sw.stats))

    peak, peak_kind = measured_peak()
    per_step = [v / args.steps for v in ph]
    qs_gbs = qb / per_step[0] / 1e9
    elems = len(sw.pts) * numel
    result = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "points": len(sw.pts), "elements_per_point": numel,
                   "phases": "quantize+pack+error reduction (fused) all -> dequantize all",
                   "launch": "one CUDA graph per phase; one grouped launch per (N, format) over "
                             "the 5 sigma tensors (14 per phase)",
                   "l2": "inputs 168 MB > 126 MB L2; sigma innermost, each buffer reused only "
                         "after >= 4 other points (>150 MB) have streamed",
                   "parallelism": f"dp{world} (independent sweeps)"},
        "phases_gbs": {"quantize_pack_stats": qs_gbs, "dequantize": db / per_step[1] / 1e9},
        "kernels_gbs": {"quantize_pack": qb / t_q / 1e9, "dequantize": db / per_step[1] / 1e9,
                        "quantize_pack_stats": qs_gbs},
        "gelem_s": {"quantize_pack_stats": elems / per_step[0] / 1e9,
                    "quantize_pack": elems / t_q / 1e9,
                    "dequantize": elems / per_step[1] / 1e9},
        "roofline": {"bound": "hbm",
                     "kernel": "fused quantize+pack+error reduction (k_qstats_small for N <= 16, "
                               "k_error_stats_bf16 for N >= 32, kStore), 14 grouped launches of 5 "
                               "tensors; per launch avg incl. its counter-reset kernel",
                     "achieved": qs_gbs, "peak": peak, "unit": "GB/s", "frac": qs_gbs / peak,
                     "peak_kind": peak_kind + " (burst copy)",
                     "traffic": FUSED_TRAFFIC_BYTES,
                     "traffic_note": "bytes per grouped launch (5 tensors, N=32), ncu "
                                     "dram__bytes_read+write; algorithmic bytes per such launch "
                                     + str(int(5 * q_bytes(numel, 32)))},
        "e2e": {"value": world * (qb + db) / e2e_s / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": args.e2e_steps, "ms_per_step": e2e_s * 1e3,
                "overlap": "double-buffered inputs: next step's H2D on a copy stream"},
        "gpu_launches": launches_per_step * args.steps,
        "deterministic_stats": deterministic,
        "small_tensor_latency_us": small,
        "wall_s_timed": t_wall,
    }
    result["clocks"] = clk.summary()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = os.cpu_count() or 1
        xs_h, rows_s, pts = oracle_sample(args.cpu_seconds, threads)
        v, dt = cpu_rate(xs_h, rows_s, pts, threads)
        result["cpu_baseline"] = {
            "value": v, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"first {rows_s} of 4096 rows of each of the 70 points, one step "
                      f"({dt:.1f} s)"}
    del graphs, g_q
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def measured_tensor_peak():
    """Dense FP4 tensor-core peak in TFLOP/s: the measured bf16 GEMM burst figure times the nominal
    FP4 : BF16 ratio of B200 (9 : 2.25)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]) * 4.0, "measured bf16 x 4 (nominal ratio)"
    except Exception:
        return 1590.0 * 4.0, "fallback bf16 x 4 (nominal ratio)"


def run_matmul_case(args):
    """Time mx_matmul (C = dequant(A) dequant(B)^T, block 16, E4M3 scales, bf16 out) on random
    codes and scales, L2 flushed before each launch; TFLOP/s = 2 m n k / median time."""
    import torch
    import fp4_microscaling_tensor_b200 as mx
    m, n, k = args.mnk
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(4096)
    a = torch.randint(0, 256, (m, k // 2), dtype=torch.uint8, device=dev, generator=g)
    b = torch.randint(0, 256, (n, k // 2), dtype=torch.uint8, device=dev, generator=g)
    sa = torch.randint(0x28, 0x48, (m, k // 16), dtype=torch.uint8, device=dev, generator=g)
    sb = torch.randint(0x28, 0x48, (n, k // 16), dtype=torch.uint8, device=dev, generator=g)
    c = torch.empty(m, n, dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)
    pa, pb = mx.prepare_scales(sa, k), mx.prepare_scales(sb, k)
    fn = lambda: mx.matmul(a, pa, b, pb, out=c, prepared=True)  # noqa: E731
    fn()
    torch.cuda.synchronize()
    times = []
    for _ in range(args.reps):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) / 1e3)
    t = statistics.median(times)
    prep = []  # the activation's scale reordering, timed alone (weights are prepared once)
    for _ in range(args.reps):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        mx.prepare_scales(sa, k, out=pa)
        e1.record()
        torch.cuda.synchronize()
        prep.append(e0.elapsed_time(e1) / 1e3)
    peak, kind = measured_tensor_peak()
    tflops = 2.0 * m * n * k / t / 1e12
    print(json.dumps({"case": "matmul", "mnk": [m, n, k], "median_us": t * 1e6, "tflops": tflops,
                      "prepare_a_scales_us": statistics.median(prep) * 1e6,
                      "frac": tflops / peak, "peak_tflops": peak, "peak_kind": kind,
                      "gave_up": mx.matmul_gave_up(), "reps": args.reps}), flush=True)


def run_case(args):
    """Time one kernel (or, with --group G, one grouped launch over G tensors) on bf16 tensors
    N(0, 0.02^2): CUDA events around each launch, L2 flushed before each launch by writing a 256 MB
    buffer; prints one JSON line."""
    import torch
    import fp4_microscaling_tensor_b200 as mx
    from fp4_microscaling_tensor_b200 import inputs
    dev = torch.device("cuda", 0)
    rows, cols = args.shape
    n, fmt, G = args.block, mx.fmt_code(args.fmt), args.group
    numel = rows * cols * G
    sets = [case_calls(args, mx, inputs, dev, r) for r in range(max(1, args.rotate))]
    code_bytes = G * rows * (((cols + 1) // 2) + -(-cols // n))  # codes + scales (any cols)
    nbytes = {"stats-recompute": numel * 2.0, "global-scale": numel * 2.0,
              "fake-quantize": numel * 4.0}.get(args.case, numel * 2.0 + code_bytes)
    fns = [c[args.case] for c in sets]
    for fn in fns:
        fn()
    torch.cuda.synchronize()
    times = []
    if args.rotate > 1:
        # one CUDA graph of 4R launches (no host gaps between them), replayed between two events
        k = 4 * len(fns)
        graph = torch.cuda.CUDAGraph()
        stream = torch.cuda.Stream()
        stream.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(stream):
            for fn in fns:  # warm-up on the capture stream
                fn()
            stream.synchronize()
            with torch.cuda.graph(graph, stream=stream):
                for j in range(k):
                    fns[j % len(fns)]()
        torch.cuda.current_stream().wait_stream(stream)
        graph.replay()
        torch.cuda.synchronize()
        for _ in range(args.reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            graph.replay()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1) / 1e3 / k)
    else:
        flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)
        for _ in range(args.reps):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fns[0]()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1) / 1e3)
    t = statistics.median(times)
    peak, kind = measured_peak()
    print(json.dumps({"case": args.case, "shape": [rows, cols], "group": G, "block": n,
                      "fmt": args.fmt, "median_us": t * 1e6, "gbs": nbytes / t / 1e9,
                      "frac": nbytes / t / 1e9 / peak, "peak": peak, "peak_kind": kind,
                      "reps": args.reps, "rotate": args.rotate}), flush=True)


def case_calls(args, mx, inputs, dev, r):
    """The calls of one input set of run_case (set r draws its tensors from seeds 100 r + k)."""
    import torch
    rows, cols = args.shape
    n, fmt, G = args.block, mx.fmt_code(args.fmt), args.group
    xs = [inputs.normal((rows, cols), 0.02, 100 * r + k, device=dev) for k in range(G)]
    if G == 1:  # (also ragged shapes, which grouped calls do not take)
        p0, s0 = mx.quantize(xs[0], n, fmt)
        packed, scales = [p0], [s0]
    else:
        packed, scales = mx.quantize_group(xs, n, fmt)
    ys = [torch.empty(rows, cols, dtype=torch.bfloat16, device=dev) for _ in range(G)]
    out = torch.empty(G, 64, dtype=torch.uint8, device=dev)
    ws = mx.stats_workspace(dev)
    if G == 1:
        x, p, sc, y = xs[0], packed[0], scales[0], ys[0]
        calls = {
            "quantize": lambda: mx.quantize(x, n, fmt, packed=p, scales=sc),
            "dequantize": lambda: mx.dequantize(p, sc, n, fmt, out=y, cols=cols),
            "stats": lambda: mx.error_stats(x, n, fmt, packed=p, scales=sc, out=out[0],
                                            workspace=ws),
            "stats-recompute": lambda: mx.error_stats(x, n, fmt, out=out[0], workspace=ws),
            "quantize-stats": lambda: mx.quantize_with_stats(x, n, fmt, packed=p, scales=sc,
                                                             out=out[0], workspace=ws),
            "global-scale": lambda: mx.global_scale(x, fmt),
            "fake-quantize": lambda: mx.fake_quantize(x, n, fmt, out=y),
        }
    else:
        calls = {
            "quantize": lambda: mx.quantize_group(xs, n, fmt, packed=packed, scales=scales),
            "dequantize": lambda: mx.dequantize_group(packed, scales, n, fmt, out=ys),
            "quantize-stats": lambda: mx.quantize_with_stats_group(
                xs, n, fmt, packed=packed, scales=scales, out=out, workspace=ws),
        }
        if args.case not in calls:
            raise SystemExit(f"--group applies to {sorted(calls)}")
    return calls


def main():
    args = parse()
    if args.case == "matmul":
        run_matmul_case(args)
        return
    if args.case:
        run_case(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
