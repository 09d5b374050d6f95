"""Benchmark of the W4A16 group-32 linear on B200.

Headline workload (one step): the decode GEMV at M = 1 over the three 4096-hidden decoder
projections (N, K) = (4096, 4096), (14336, 4096), (4096, 14336), with RTN group-32 signed
int4 codes and fp32 scales quantized on the GPU from W ~ N(0, 0.02^2) and bf16 x ~ N(0, 1).
Metric: weight GB/s = packed payload bytes (codes + 4 * scales, the LoopQ payload_bytes)
per second. Four rotating copies of the weights (336 MB > 126 MB L2) make every step read
weights last touched three steps earlier, so L2 cannot serve them.

The timed steps run as CUDA graphs replayed back to back with CUDA events around the
replays; every launch in the timed region is the GEMV, so its mean duration is the region
time per launch (inter-launch gaps included). The
JSON line also carries the end-to-end number (public Python API, pinned host x in, y out
every step), the roofline of the GEMV kernel, the oracle timed on the host cores, and a
per-workload detail block (odd-width dequant, batched decode, prefill TFLOP/s, asymmetric
act-order, quantize).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun every rank runs an independent replica (no collective on the data path);
value = units processed by all ranks / max-over-ranks time.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "W4A16 group-32 linear: weight GB/s (% of HBM peak) decode; TFLOP/s prefill"
UNIT = "GB/s"
L2_BYTES = 126 * 1024 * 1024
ROTATE = 4
GRAPH_CHUNK = 1000  # steps per captured graph


WARM_SECONDS = 0.3  # untimed load before the timed regions
REGION_TARGET_S = 0.5  # total time of the repeated timed regions (at least MIN_REPEATS)
MIN_REPEATS, MAX_REPEATS = 5, 51


def repeats(steps, est_us_per_step=25.0):
    """How many times the K-step timed region is repeated: enough regions to give a median
    and p10/p90, about REGION_TARGET_S seconds in all."""
    n = int(REGION_TARGET_S / max(steps * est_us_per_step * 1e-6, 1e-9))
    return max(MIN_REPEATS, min(MAX_REPEATS, n))


def spread(values):
    """Median, p10 and p90 (linear interpolation) of a list of region times."""
    v = np.sort(np.asarray(values, dtype=np.float64))
    return {"median": float(np.median(v)), "p10": float(np.percentile(v, 10)),
            "p90": float(np.percentile(v, 90)), "n": int(v.size)}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def payload(N, K):
    return N * ((K + 1) // 2) + 4 * N * ((K + 31) // 32)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def recorded_traffic(kernel_file, summary):
    """Per-launch DRAM traffic of the GEMV from the committed ncu summary, or None when the
    kernel source changed after the counters were taken."""
    try:
        text = open(os.path.join(ROOT, "profiles", summary)).read()
        src = open(os.path.join(ROOT, "weight_only_int4_04_b200", "csrc", kernel_file), "rb").read()
    except OSError:
        return None
    m = re.search(r"bench-traffic: sha256=([0-9a-f]+) bytes_per_step_launch_mean=([0-9.e+]+)", text)
    if not m or m.group(1) != hashlib.sha256(src).hexdigest()[:16]:
        return None
    return float(m.group(2))


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, uuid):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-i", uuid,
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        self.t0 = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], [], set()
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle as it stands
# ---------------------------------------------------------------------------

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [int(i.get("num_threads", 1)) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_sample(frac_rows=8):
    """One bounded sample of the decode workload for the oracle: 1/frac_rows of the rows of
    each of the three shapes (all K). Returns (callable, payload bytes per call, text)."""
    import oracle as O
    cases = []
    for N, K in workloads.DECODE_SHAPES:
        c = workloads.decode_case(N, K)
        n = N // frac_rows
        q, s = O.quantize_rtn(c["W"][:n])
        cases.append((c["x"], O.pack_nibbles(q), s, K))

    def run():
        for x, codes, s, K in cases:
            O.linear(x, codes, s, K)
    nbytes = sum(payload(N // frac_rows, K) for N, K in workloads.DECODE_SHAPES)
    return run, nbytes, f"oracle linear (dequantize + fp64 matmul) at M=1 on 1/{frac_rows} of the rows of each decode shape"


def oracle_detail_samples(frac_rows=8):
    """Bounded oracle samples for the detail rows that have a host-side baseline: name ->
    (callable, payload bytes per call, text). 1/frac_rows of the rows of each shape."""
    import oracle as O
    import oracle.q4_0 as Q
    out = {}
    q4 = []
    for N, K in workloads.Q4_0_SHAPES:
        c = workloads.q4_0_case(N + K, 1, N, K, bias=False)
        q4.append((c["x"], c["blocks"][: N // frac_rows], K))

    def run_q4():
        for x, blocks, K in q4:
            Q.linear(x, blocks, K)
    out["q4_0_decode_M1_step"] = (run_q4, sum(Q.payload_bytes(N // frac_rows, K) for N, K in workloads.Q4_0_SHAPES),
                                  f"oracle Q4_0 linear at M=1 on 1/{frac_rows} of the rows of each decode shape")
    N, K = workloads.BATCHED_SHAPE
    c = workloads.decode_case(N, K, M=1, config=3)
    n = N // frac_rows
    q, sc = O.quantize_rtn(c["W"][:n])
    codes = O.pack_nibbles(q)
    _, dy = workloads.draw_x(np.random.default_rng([3, 1]), 1, n)

    def run_bwd():
        O.linear_backward_x(dy, codes, sc, K)
    out["backward_x_M1_14336x4096"] = (run_bwd, payload(n, K) + 2 * n + 2 * K,
                                       f"oracle input gradient at M=1 on 1/{frac_rows} of the rows of (14336,4096)")
    return out


def time_oracle(run, nbytes, text, seconds=3.0):
    """The oracle's throughput on one bounded sample (GB/s of the sample's payload)."""
    try:
        run()
        t0 = time.perf_counter()
        reps = 0
        while True:
            run()
            reps += 1
            if time.perf_counter() - t0 > seconds:
                break
        dt = time.perf_counter() - t0
        return {"value": reps * nbytes / dt / 1e9, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
                "sample": text + f"; {reps} repetitions in {dt:.1f} s"}
    except Exception as e:  # a failed baseline is reported, it does not stop the bench
        return {"value": None, "unit": "GB/s", "kind": "oracle", "error": str(e)[:200]}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    run, nbytes, text = oracle_sample()
    for _ in range(max(args.warmup, 0)):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = time.perf_counter() - t0
    value = args.steps * nbytes / dt / 1e9
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "decode GEMV M=1, (N,K) in (4096,4096),(14336,4096),(4096,14336); sampled rows",
                   "sample": text, "l2": "n/a (host)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": text},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def max_over_ranks(x: float, device) -> float:
    """The largest of every rank's `x` (the time of a replicated step is the slowest
    rank's); `x` itself with a single process. `device`: where the backend's tensors live
    (a CUDA device for NCCL, the CPU for gloo)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(units_per_rank: float, world: int, ms: float) -> float:
    """Whole-job throughput: the units every replica processed over the slowest rank's time
    (GB/s for bytes and milliseconds)."""
    return world * units_per_rank / (ms * 1e-3) / 1e9


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=100)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-detail", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--only", default=None,
                    help="time one named detail workload (e.g. prefill_4096x14336x4096) and exit")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    import weight_only_int4_04_b200 as w4  # fails loudly without the built library
    # The decode weights are written once, before any timed work (and synchronized), so the
    # decode GEMVs may stream them before the previous kernel of the stream has finished.
    w4.set_weight_prefetch(True)

    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    if args.only is not None:
        hbm_peak, tc_peak, _, _ = peaks()
        res = run_detail(w4, dev, hbm_peak, tc_peak, only=args.only, iters=args.steps, warmup=args.warmup)
        if not res:
            raise SystemExit(f"unknown workload {args.only}")
        print(json.dumps({"only": args.only, **res[args.only]}), flush=True)
        return 0

    # -- workload: three decode shapes, quantized by the library, 4 rotating copies ------
    shapes = workloads.DECODE_SHAPES
    sets, xs, ys = [], [], []
    for N, K in shapes:
        c = workloads.decode_case(N, K)
        W = torch.from_numpy(c["W"]).to(dev)
        codes, scales = w4.quantize_rtn(W)
        del W
        sets.append([(codes.clone(), scales.clone()) for _ in range(ROTATE)])
        xs.append(torch.from_numpy(c["x_bits"].view(np.int16)).to(dev).view(torch.bfloat16))
        ys.append(torch.empty((1, N), dtype=torch.bfloat16, device=dev))
    step_bytes = sum(payload(N, K) for N, K in shapes)
    algo_bytes = [payload(N, K) + 2 * K + 2 * N for N, K in shapes]  # weights + x + y per launch

    def step(i):
        r = i % ROTATE
        for j, (N, K) in enumerate(shapes):
            codes, scales = sets[j][r]
            w4.linear(xs[j], codes, scales, K, out=ys[j])

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    # -- capture the timed steps as CUDA graphs of up to GRAPH_CHUNK steps. No event nodes
    # inside the graphs: an event node between launches costs ~4-5 us of GPU time, more than
    # a small GEMV itself, so the step is timed by events around the replays and the kernel
    # time per launch is the timed region divided by the launches (all of them GEMVs).
    graphs = []
    side = torch.cuda.Stream()
    done = 0
    while done < args.steps:
        n = min(GRAPH_CHUNK, args.steps - done)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            for i in range(n):
                step(done + i)
        graphs.append(g)
        done += n
    torch.cuda.synchronize()
    graphs[0].replay()  # first replay uploads the graph; not part of the timing
    torch.cuda.synchronize()

    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid)
    # untimed load until the clocks have settled (an idle GPU needs some time to ramp up)
    t_w = time.perf_counter()
    while time.perf_counter() - t_w < WARM_SECONDS:
        for g in graphs:
            g.replay()
        torch.cuda.synchronize()
    # the K timed steps, R times over: each region is exactly the K steps, bracketed by a
    # barrier and a synchronize on both sides; the line reports the median region
    region_ms = []
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    for _ in range(repeats(args.steps)):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t_start.record(stream)
        for g in graphs:
            g.replay()
        t_end.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        region_ms.append(max_over_ranks(t_start.elapsed_time(t_end), dev))
    clocks = sampler.stop()
    dist_ms = spread(region_ms)
    ms = dist_ms["median"]

    launches = args.steps * len(shapes)
    hbm_peak, tc_peak, tc_sus, peak_kind = peaks()
    # every launch of the timed region is the GEMV kernel: its average duration is the
    # region time per launch (graph launch gaps included, so this is conservative)
    achieved = args.steps * sum(algo_bytes) / (ms * 1e-3) / 1e9
    value = job_value(args.steps * step_bytes, world, ms)

    # per-shape split, measured the same way on graphs of one shape (reported, not timed region)
    per_shape_us = {}
    for j, (N, K) in enumerate(shapes):
        reps = 200
        gj = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gj, stream=side):
            for i in range(reps):
                codes, scales = sets[j][i % ROTATE]
                w4.linear(xs[j], codes, scales, K, out=ys[j])
        gj.replay()
        torch.cuda.synchronize()
        a_ev, b_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_ev.record(stream)
        gj.replay()
        b_ev.record(stream)
        torch.cuda.synchronize()
        per_shape_us[f"{N}x{K}"] = 1e3 * a_ev.elapsed_time(b_ev) / reps
        del gj

    # -- end to end through the public API: pinned x in, y out, every step --------------
    # The step's three activation rows travel in one pinned host buffer (one copy in) and
    # the three outputs come back in one (one copy out), as a caller batching a step would.
    e2e_steps = min(args.steps, 5000)
    x_sizes = [x.numel() for x in xs]
    y_sizes = [y.numel() for y in ys]
    hx_all = torch.cat([x.reshape(-1).cpu() for x in xs]).pin_memory()
    hy_all = torch.empty(sum(y_sizes), dtype=torch.bfloat16).pin_memory()
    dx_all = torch.empty(sum(x_sizes), dtype=torch.bfloat16, device=dev)
    dy_all = torch.empty(sum(y_sizes), dtype=torch.bfloat16, device=dev)
    dx = [t.view(1, -1) for t in torch.split(dx_all, x_sizes)]
    dy = [t.view(1, -1) for t in torch.split(dy_all, y_sizes)]
    h2d = hx_all.numel() * 2
    d2h = hy_all.numel() * 2

    # the layers as a caller holds them: prepared once, called every step
    layers = [[w4.Linear(c, s, K=K) for c, s in sets[j]] for j, (N, K) in enumerate(shapes)]

    def e2e_step(i):
        r = i % ROTATE
        dx_all.copy_(hx_all, non_blocking=True)
        for j in range(len(shapes)):
            layers[j][r](dx[j], out=dy[j])
        hy_all.copy_(dy_all, non_blocking=True)

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(e2e_steps):
        e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    e2e_value = job_value(e2e_steps * step_bytes, world, e2e_ms)

    detail = None
    if rank == 0 and not args.no_detail:
        detail = run_detail(w4, dev, hbm_peak, tc_peak)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        run, nbytes, text = oracle_sample()
        run()
        t0 = time.perf_counter()
        reps = 0
        while True:
            run()
            reps += 1
            if time.perf_counter() - t0 > 10.0:
                break
        dt = time.perf_counter() - t0
        cpu = {"value": reps * nbytes / dt / 1e9, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": text + f"; {reps} repetitions in {dt:.1f} s on {os.cpu_count()} host CPUs",
               "cpu_model": cpu_model(), "host_cpus": os.cpu_count()}
        try:  # the same sample on one thread
            from threadpoolctl import threadpool_limits
            with threadpool_limits(limits=1):
                run()
                t0 = time.perf_counter()
                reps1 = 0
                while True:
                    run()
                    reps1 += 1
                    if time.perf_counter() - t0 > 5.0:
                        break
                dt1 = time.perf_counter() - t0
            cpu["single_thread"] = {"value": reps1 * nbytes / dt1 / 1e9, "unit": UNIT, "cores": 1,
                                    "sample": text + f"; {reps1} repetitions in {dt1:.1f} s"}
        except Exception as e:
            cpu["single_thread"] = {"value": None, "error": str(e)[:200]}
        if detail is not None:
            try:
                samples = oracle_detail_samples()
            except Exception as e:
                samples = {}
                for name in ("q4_0_decode_M1_step", "backward_x_M1_14336x4096"):
                    if name in detail:
                        detail[name]["cpu_baseline"] = {"value": None, "kind": "oracle", "error": str(e)[:200]}
            for name, (run_d, nb_d, text_d) in samples.items():
                if name in detail:
                    detail[name]["cpu_baseline"] = time_oracle(run_d, nb_d, text_d)

    if world > 1:
        dist.barrier()
        for g in graphs:
            del g
        graphs.clear()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    frac = achieved / hbm_peak
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 x int4 -> fp32", "data": "synthetic",
        "config": {"workload": "decode GEMV M=1: (N,K) = (4096,4096), (14336,4096), (4096,14336); "
                               "RTN group-32 int4 + fp32 scales from W~N(0,0.02^2); x bf16 ~N(0,1); no bias",
                   "l2": f"inputs larger than L2: {ROTATE} rotating weight copies, {ROTATE * step_bytes / 2**20:.0f} MiB",
                   "timing": "CUDA graphs of <=1000 steps replayed back to back, CUDA events on the launching stream "
                             f"around the replays; {WARM_SECONDS} s of untimed replays first; the K-step region "
                             f"timed {dist_ms['n']} times (barrier + synchronize around each), value from the median",
                   "launch": "programmatic dependent launch; weights prefetched before the previous GEMV ends (weights constant)",
                   "parallelism": f"replicas x{world}"},
        "clocks": clocks,
        "region_ms": {k: dist_ms[k] for k in ("median", "p10", "p90", "n")},
        "value_p10_p90": [job_value(args.steps * step_bytes, world, dist_ms["p90"]),
                          job_value(args.steps * step_bytes, world, dist_ms["p10"])],
        "gpu_launches": launches,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps,
                "note": "public Python API per step (w4.Linear, prepared once per weight copy): one "
                        "pinned-host copy of the step's three x rows to the device, 3 linears, one copy of the "
                        "three y rows to pinned host; weights resident in HBM"},
        "roofline": {"bound": "hbm", "kernel": "gemv_tma_kernel (M=1 decode GEMV)", "achieved": achieved, "peak": hbm_peak,
                     "unit": "GB/s", "frac": frac, "peak_kind": peak_kind,
                     "traffic": recorded_traffic("k_gemv_tma.cu", "gemv_tma_decode_m1.md"),
                     "algorithmic_bytes_per_step": sum(algo_bytes),
                     "launch_us_mean": 1e3 * ms / launches,
                     "per_shape_gbs": {f"{N}x{K}": b / us / 1e3
                                       for (N, K), b, us in zip(shapes, algo_bytes, per_shape_us.values())},
                     "per_shape_us": per_shape_us},
        "cpu_baseline": cpu,
        "detail": detail,
    }
    print(json.dumps(line), flush=True)
    return 0


def detail_workloads(w4, dev, hbm_peak, tc_peak):
    """Named workloads of the other configurations. Each entry builds its inputs and returns
    (calls, report): calls cycle through ROTATE weight copies (so that no launch finds its
    weights in L2) and report(us) gives the line's figures."""
    import torch

    def bf16(bits):
        return torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)

    def dequant_odd():
        N, K = workloads.ODD_DEQUANT_SHAPE
        c = workloads.decode_case(N, K)
        codes, scales = w4.quantize_rtn(torch.from_numpy(c["W"]).to(dev))
        copies = [(codes.clone(), scales.clone()) for _ in range(ROTATE)]
        o = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
        nb = payload(N, K) + 2 * N * K
        return ([lambda c=c, s=s: w4.dequantize(c, s, K, torch.bfloat16, out=o) for c, s in copies],
                lambda us: {"us": us, "gbs": nb / us / 1e3, "frac_hbm": nb / us / 1e3 / hbm_peak})

    def quantize():
        N, K = workloads.BATCHED_SHAPE
        c = workloads.decode_case(N, K, M=1, config=3, bias=True)
        W = torch.from_numpy(c["W"]).to(dev)  # 235 MB of fp32 input: larger than L2 by itself
        st = torch.zeros(1, dtype=torch.int32, device=dev)
        codes = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty((N, K // 32), dtype=torch.float32, device=dev)
        nb = 4 * N * K + payload(N, K)
        return ([lambda: w4.quantize_rtn(W, status=st, out=(codes, scales))],
                lambda us: {"us": us, "gbs": nb / us / 1e3, "frac_hbm": nb / us / 1e3 / hbm_peak})

    def batched(M):
        def make():
            N, K = workloads.BATCHED_SHAPE
            c = workloads.decode_case(N, K, M=M, config=3, bias=True)
            codes, scales = w4.quantize_rtn(torch.from_numpy(c["W"]).to(dev))
            copies = [(codes.clone(), scales.clone()) for _ in range(ROTATE)]
            bias = torch.from_numpy(c["bias"]).to(dev)
            x = bf16(c["x_bits"])
            y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            fl = 2.0 * M * N * K
            return ([lambda c=c, s=s: w4.linear(x, c, s, K, bias=bias, out=y) for c, s in copies],
                    lambda us: {"us": us, "weight_gbs": payload(N, K) / us / 1e3,
                                "frac_hbm": payload(N, K) / us / 1e3 / hbm_peak, "tflops": fl / us / 1e6,
                                "frac_tensor": fl / us / 1e6 / tc_peak})
        return make

    def prefill(M, N, K):
        def make():
            c = workloads.decode_case(N, K, M=M, config=4)
            codes, scales = w4.quantize_rtn(torch.from_numpy(c["W"]).to(dev))
            x = bf16(c["x_bits"])
            y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            fl = 2.0 * M * N * K
            return ([lambda: w4.linear(x, codes, scales, K, out=y)],
                    lambda us: {"us": us, "tflops": fl / us / 1e6, "frac_tensor": fl / us / 1e6 / tc_peak})
        return make

    def asym(M):
        def make():
            a = workloads.asym_random_codes(M)
            gi = torch.from_numpy(a["g_idx"]).to(dev)
            sc, perm = w4.asym_prepare(torch.from_numpy(a["codes"]).to(dev), gi, a["K"], a["n_groups"])
            s = torch.from_numpy(a["scales"]).to(dev)
            z = torch.from_numpy(a["zeros"]).to(dev)
            copies = [(sc.clone(), s.clone(), z.clone()) for _ in range(ROTATE)]
            x = bf16(a["x_bits"])
            b = torch.from_numpy(a["bias"]).to(dev)
            y = torch.empty((M, a["N"]), dtype=torch.bfloat16, device=dev)
            need = w4.asym_workspace_bytes(M, a["N"], a["K"], a["n_groups"])
            ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev) if need else None
            nb = a["codes"].size + 4 * a["scales"].size + a["zeros"].size + 4 * a["K"]
            fl = 2.0 * M * a["N"] * a["K"]
            return ([lambda c=c, s_=s_, z_=z_: w4.linear_asym_gidx(x, c, s_, z_, gi, perm=perm, bias=b, out=y,
                                                                   workspace=ws) for c, s_, z_ in copies],
                    lambda us: {"us": us, "weight_gbs": nb / us / 1e3, "frac_hbm": nb / us / 1e3 / hbm_peak,
                                "tflops": fl / us / 1e6, "frac_tensor": fl / us / 1e6 / tc_peak,
                                "bound": "hbm" if M <= 16 else "tensor"})
        return make

    def q4_0_decode():
        # the headline's decode step on GGUF Q4_0 blocks (18 bytes per 32 weights): one call
        # = the three projections in turn, each on its own rotating block copy
        sets, xs, ys, nb = [], [], [], 0
        for N, K in workloads.Q4_0_SHAPES:
            c = workloads.q4_0_case(N + K, 1, N, K, bias=False)
            blk = torch.from_numpy(c["blocks"]).to(dev)
            sets.append([blk.clone() for _ in range(ROTATE)])
            xs.append(bf16(c["x_bits"]))
            ys.append(torch.empty((1, N), dtype=torch.bfloat16, device=dev))
            nb += N * (K // 32) * 18

        def step(r):
            for j in range(len(xs)):
                w4.linear_q4_0(xs[j], sets[j][r], out=ys[j])
        return ([lambda r=r: step(r) for r in range(ROTATE)],
                lambda us: {"us": us, "weight_gbs": nb / us / 1e3, "frac_hbm": nb / us / 1e3 / hbm_peak})

    def q4_0_as_group32_decode():
        # the same Q4_0 decode step after a one-time re-layout of every block copy into the
        # group-32 format (w4_q4_0_to_group32, outside the timed region): the group-32 decode
        # GEMV then streams 20 bytes per 32 weights. Throughput is counted in the blocks'
        # 18 bytes per 32 weights, so that the row compares with q4_0_decode_M1_step;
        # stream_gbs counts the bytes actually read
        sets, xs, ys, nb, ns = [], [], [], 0, 0
        for N, K in workloads.Q4_0_SHAPES:
            c = workloads.q4_0_case(N + K, 1, N, K, bias=False)
            blk = torch.from_numpy(c["blocks"]).to(dev)
            sets.append([w4.Linear(*w4.q4_0_to_group32(blk, K), None, K) for _ in range(ROTATE)])
            xs.append(bf16(c["x_bits"]))
            ys.append(torch.empty((1, N), dtype=torch.bfloat16, device=dev))
            nb += N * (K // 32) * 18
            ns += payload(N, K)

        def step(r):
            for j in range(len(xs)):
                sets[j][r](xs[j], out=ys[j])
        return ([lambda r=r: step(r) for r in range(ROTATE)],
                lambda us: {"us": us, "weight_gbs": nb / us / 1e3, "frac_hbm": nb / us / 1e3 / hbm_peak,
                            "stream_gbs": ns / us / 1e3})

    def channel_decode():
        # the headline's decode step on per-channel weights (one fp32 scale per row, read by
        # the decode kernel: 0.5 bytes per weight + 4 per row)
        sets, xs, ys, nb = [], [], [], 0
        for N, K in workloads.DECODE_SHAPES:
            c = workloads.decode_case(N, K)
            codes, scales = w4.quantize_rtn_channel(torch.from_numpy(c["W"]).to(dev))
            sets.append([(codes.clone(), scales.clone()) for _ in range(ROTATE)])
            xs.append(bf16(c["x_bits"]))
            ys.append(torch.empty((1, N), dtype=torch.bfloat16, device=dev))
            nb += N * ((K + 1) // 2) + 4 * N

        def step(r):
            for j, (N, K) in enumerate(workloads.DECODE_SHAPES):
                cd, sc = sets[j][r]
                w4.linear_channel(xs[j], cd, sc, K, out=ys[j])
        return ([lambda r=r: step(r) for r in range(ROTATE)],
                lambda us: {"us": us, "weight_gbs": nb / us / 1e3, "frac_hbm": nb / us / 1e3 / hbm_peak})

    def lora_merge(r):
        # merge a rank-r adapter into the (14336, 4096) projection and re-quantize it (an offline
        # call): codes and scales read and written (separate output copies, so that every call
        # merges the same weight), the two factors read once
        def make():
            N, K = workloads.BATCHED_SHAPE
            c = workloads.decode_case(N, K, M=1, config=3)
            codes, scales = w4.quantize_rtn(torch.from_numpy(c["W"]).to(dev))
            copies = [(codes.clone(), scales.clone()) for _ in range(ROTATE)]
            g = torch.Generator(device="cpu").manual_seed(11)
            bt = (torch.randn(N, r, generator=g) * 0.01).to(dev)
            at = (torch.randn(r, K, generator=g) * 0.01).to(dev)
            outs = [(torch.empty_like(codes), torch.empty_like(scales)) for _ in range(ROTATE)]
            st = torch.zeros(1, dtype=torch.int32, device=dev)
            nb = 2 * payload(N, K) + 4 * r * (N + K)
            # the rank sum is r separately rounded products and r sums per weight in scalar fp32,
            # so the call is bound by fp32 issue: 148 SMs x 128 lanes x the 1965 MHz maximum clock
            ops = 2 * N * K * r
            fp32_peak = 148 * 128 * 1.965e9
            return ([lambda c=c, s=s, o=o: w4.lora_merge(c, s, K, bt, at, 2.0, out=o, status=st)
                     for (c, s), o in zip(copies, outs)],
                    lambda us: {"us": us, "gbs": nb / us / 1e3, "frac_hbm": nb / us / 1e3 / hbm_peak,
                                "fp32_tops": ops / us / 1e6, "frac_fp32": ops / (us * 1e-6) / fp32_peak,
                                "rank": r})
        return make

    def backward_x(M):
        # input gradient dx = dy . dequant(W) of the (14336, 4096) projection
        def make():
            N, K = workloads.BATCHED_SHAPE
            c = workloads.decode_case(N, K, M=1, config=3)
            codes, scales = w4.quantize_rtn(torch.from_numpy(c["W"]).to(dev))
            copies = [(codes.clone(), scales.clone()) for _ in range(ROTATE)]
            dy_bits, _ = workloads.draw_x(np.random.default_rng([3, M]), M, N)
            dy = bf16(dy_bits)
            dx = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
            need = int(w4.lib.w4_linear_backward_x_workspace_bytes(M, N, K))
            ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
            nb = payload(N, K) + 2 * M * N + 2 * M * K
            return ([lambda c=c, s=s: w4.linear_backward_x(dy, c, s, K, out=dx, workspace=ws) for c, s in copies],
                    lambda us: {"us": us, "gbs": nb / us / 1e3, "frac_hbm": nb / us / 1e3 / hbm_peak})
        return make

    w = {"dequant_4096x4095_bf16": dequant_odd, "quantize_14336x4096": quantize, "q4_0_decode_M1_step": q4_0_decode,
         "q4_0_as_group32_decode_M1_step": q4_0_as_group32_decode,
         "channel_decode_M1_step": channel_decode, "lora_merge_r16_14336x4096": lora_merge(16),
         "backward_x_M1_14336x4096": backward_x(1), "backward_x_M16_14336x4096": backward_x(16)}
    for M in workloads.BATCHED_M:
        w[f"batched_M{M}_14336x4096"] = batched(M)
    for M, N, K in workloads.PREFILL_SHAPES:
        w[f"prefill_{M}x{N}x{K}"] = prefill(M, N, K)
    for M in workloads.ASYM_M:
        w[f"asym_M{M}_11008x4096_g128"] = asym(M)
    return w


def run_detail(w4, dev, hbm_peak, tc_peak, only=None, iters=None, warmup=2):
    """Time each named workload the way the headline is timed: a CUDA graph of back-to-back
    calls cycling through rotating weight copies, CUDA events around one replay; the time per
    call is the replay time divided by the calls."""
    import torch

    out = {}
    side = torch.cuda.Stream()
    for name, make in detail_workloads(w4, dev, hbm_peak, tc_peak).items():
        if only is not None and name != only:
            continue
        calls, report = make()
        reps = iters if iters is not None else (10 if name.startswith("prefill") else 100)
        for i in range(max(warmup, len(calls))):
            calls[i % len(calls)]()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            for i in range(reps):
                calls[i % len(calls)]()
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        out[name] = report(1e3 * a.elapsed_time(b) / reps)
        del g, calls
        torch.cuda.empty_cache()
    return out


if __name__ == "__main__":
    sys.exit(main())
