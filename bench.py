"""Benchmark of the dynamic-FP8 hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload large|large4096|sweep|moe]

Default workload (the large a8w8 GEMM layer): X bf16 [16384, 8192] ~N(0,1),
W bf16 [28672, 8192] ~N(0,0.02).  One step = per-token E4M3 quantize of X,
per-output-channel E4M3 quantize of W (one scale per row of W[N,K]), and the
a8w8 GEMM into a caller-owned bf16 out [16384, 28672].  Inputs are larger
than L2 (126 MB), so no flush is needed between steps.  Metric: TFLOP/s of
the GEMM's 2*M*N*K per step time; the quantize kernels' GB/s is reported
beside it.  Multi-GPU (torchrun): each rank runs the same step on its own
tokens with replicated weights (data parallel, no collective in the data
path); the timed region is the max over ranks.

--impl reference times the CPU oracle (the plain C reference) on a bounded
sample of the same workload per step, on the host cores.
"""
import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_OVER_BF16 = 4.5 / 2.25  # nominal dense ratio (fp8 4.5 PF vs bf16 2.25 PF)
METRIC = "a8w8 GEMM TFLOP/s and quantize GB/s, as % of B200 FP8 / HBM roofline"


def load_peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return FALLBACK, "fallback"


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


# --------------------------------------------------------------- workloads
WORKLOADS = {
    "large": dict(M=16384, N=28672, K=8192),
    "large4096": dict(M=4096, N=28672, K=8192),
}


def workload_desc(name, cfg):
    if name.startswith("large"):
        return ("large a8w8 GEMM layer: X bf16 [%d,%d] ~N(0,1) per-token E4M3, W bf16 [%d,%d] ~N(0,0.02) "
                "per-output-channel E4M3, out bf16 [%d,%d] (caller-owned)" % (cfg["M"], cfg["K"], cfg["N"],
                                                                            cfg["K"], cfg["M"], cfg["N"]))
    return name


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        self.proc.wait()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        power = [float(r[3]) for r in rows if re.match(r"^[0-9.]+$", r[3])]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        # samples under load: the upper half of the power readings
        loaded = sm
        if power and len(power) == len(sm):
            cut = statistics.median(power)
            loaded = [s for s, p in zip(sm, power) if p >= cut] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows),
                "power_w_max": max(power) if power else None}


def traffic_from_profile(kernel_file, profile_name):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel source changed since the capture."""
    path = os.path.join(ROOT, "profiles", profile_name)
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    h = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
    if not m or not h:
        return None
    src = os.path.join(ROOT, "fp8_dynamic_quantization_amax_b200", "csrc", kernel_file)
    cur = hashlib.sha256(open(src, "rb").read()).hexdigest()
    return float(m.group(1)) if cur == h.group(1) else None


# ------------------------------------------------------------ rank logic
def max_over_ranks(ms, world, device):
    """The timed region of a multi-rank run is the slowest rank's."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_step, steps, world, max_ms):
    """Whole-job throughput: every rank's work over the slowest rank's time."""
    return flops_per_step * steps * world / (max_ms / 1e3) / 1e12


# ------------------------------------------------------------------ ours
def run_ours(args, rank, local_rank, world):
    import torch
    import torch.distributed as dist

    import workloads as W
    import fp8_dynamic_quantization_amax_b200 as hq

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    cfg = WORKLOADS[args.workload]
    M, N, K = cfg["M"], cfg["N"], cfg["K"]
    peaks, peak_src = load_peaks()

    # inputs: seeded host generation; tokens differ per rank, weights replicated
    x_bits = W.large_x(M, K, seed=rank)
    w_bits = W.large_w(N, K)
    x_host = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    w_host = torch.from_numpy(w_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    x = x_host.to(dev).view(M, K)
    w = w_host.to(dev).view(N, K)
    xq = torch.empty((M, K), dtype=torch.uint8, device=dev)
    wq = torch.empty((N, K), dtype=torch.uint8, device=dev)
    xs = torch.empty((M,), dtype=torch.float32, device=dev)
    ws = torch.empty((N,), dtype=torch.float32, device=dev)
    out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        hq.hq_quantize_fp8(x, hq.E4M3, hq.PER_TOKEN, q=xq, scales=xs, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        hq.hq_quantize_fp8(w, hq.E4M3, hq.PER_TOKEN, q=wq, scales=ws, stream=stream)
        if ev is not None:
            ev[2].record(stream)
        hq.hq_gemm_a8w8(xq, wq, xs, ws, hq.E4M3, out=out, stream=stream)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    hq.hq_check_device_error()

    clocks = ClockSampler(local_rank)
    clocks.start()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    hq.hq_check_device_error()
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    qx_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    qw_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    g_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)

    flops = 2.0 * M * N * K
    value = whole_job_tflops(flops, args.steps, world, ms)
    gemm_tflops = flops / (g_ms / 1e3) / 1e12
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    q_bytes_x = M * K * 3 + M * 4  # bf16 read, code write, f32 scale write
    q_bytes_w = N * K * 3 + N * 4
    qx_gbs = q_bytes_x / (qx_ms / 1e3) / 1e9
    qw_gbs = q_bytes_w / (qw_ms / 1e3) / 1e9

    # end to end through the C ABI with host buffers: H2D of X and W, the
    # three kernels, D2H of out, every step
    out_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(1, min(args.steps, 5))

    def e2e_step():
        x.copy_(x_host, non_blocking=True)
        w.copy_(w_host, non_blocking=True)
        step()
        out_host.copy_(out, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = whole_job_tflops(flops, e2e_steps, world, e2e_ms)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(M, N, K, budget_rows=(256, 4096))

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    traffic = traffic_from_profile("gemm.cu", "gemm_a8w8_large_M16384_N28672_K8192.md") \
        if args.workload == "large" else None
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8_e4m3 (fp32 accumulate, bf16 out)",
        "data": "synthetic (seeded host normals; X seed = rank, W seed 1)",
        "config": {"workload": workload_desc(args.workload, cfg), "M": M, "N": N, "K": K,
                   "l2": "inputs larger than L2 (X %d MB, W %d MB, out %d MB); no flush" %
                         (M * K * 2 >> 20, N * K * 2 >> 20, M * N * 2 >> 20),
                   "parallelism": "dp%d" % world},
        "roofline": {"bound": "tensor", "achieved": round(gemm_tflops, 1), "peak": round(fp8_peak, 1),
                     "unit": "TFLOP/s", "frac": round(gemm_tflops / fp8_peak, 4), "traffic": traffic,
                     "kernel": "k_gemm2<fp8, 256x256 CTA pair> (tcgen05 cta_group::2 kind::f8f6f4)",
                     "peak_source": "%s bf16 burst %.1f TFLOP/s x %.0f (nominal fp8/bf16 dense ratio)" %
                                    (peak_src, peaks["bf16_tflops"], FP8_OVER_BF16)},
        "quantize": {"x_per_token": {"ms": round(qx_ms, 4), "GB/s": round(qx_gbs, 1),
                                     "frac_hbm": round(qx_gbs / peaks["hbm_gbs"], 4)},
                     "w_per_channel": {"ms": round(qw_ms, 4), "GB/s": round(qw_gbs, 1),
                                       "frac_hbm": round(qw_gbs / peaks["hbm_gbs"], 4)},
                     "bytes": "algorithmic: 2 B read + 1 B write per element + 4 B per scale",
                     "hbm_peak_gbs": peaks["hbm_gbs"], "peak_source": peak_src},
        "gemm_ms": round(g_ms, 4),
        "clocks": clk,
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": (M * K + N * K) * 2, "d2h_bytes_per_step": M * N * 2,
                "steps": e2e_steps},
        "gpu_launches": 3 * args.steps,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line))


# --------------------------------------------------------------- oracle
def cpu_baseline(M, N, K, budget_rows, seed=0):
    """The oracle, as it stands, on a bounded sample of the workload: per-token
    quantize of `mx` rows of X and `nw` rows of W, then the exact GEMM of the
    sample.  Returns TFLOP/s of the sample's GEMM flops per oracle time."""
    import oracle as O
    import workloads as W
    mx, nw = budget_rows
    rng = np.random.default_rng(seed)
    x = W.f32_to_bf16_bits(rng.standard_normal((mx, K), dtype=np.float32))
    w = W.f32_to_bf16_bits(rng.standard_normal((nw, K), dtype=np.float32) * np.float32(0.02))
    O.lib()
    t = time.perf_counter()
    xq, xs, _ = O.quantize(x, O.E4M3, O.PER_TOKEN)
    wq, ws, _ = O.quantize(w, O.E4M3, O.PER_TOKEN)
    O.gemm_a8w8(xq, wq, O.E4M3, xs, ws)
    dt = time.perf_counter() - t
    flops = 2.0 * mx * nw * K
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
            "sample": "X %d rows x W %d rows (K=%d): per-token quantize of both + exact GEMM, %.1f s"
                      % (mx, nw, K, dt),
            "seconds": round(dt, 2)}


def run_reference(args, rank, world):
    if rank != 0:
        return
    cfg = WORKLOADS[args.workload]
    M, N, K = cfg["M"], cfg["N"], cfg["K"]
    rows = (8, 512)
    for _ in range(args.warmup):
        cpu_baseline(M, N, K, rows)
    t = time.perf_counter()
    last = None
    for i in range(args.steps):
        last = cpu_baseline(M, N, K, rows, seed=i)
    dt = time.perf_counter() - t
    flops = 2.0 * rows[0] * rows[1] * K
    value = flops * args.steps / dt / 1e12
    line = {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt * 1e3 / max(args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp8_e4m3 codes, exact integer GEMM, f64",
        "data": "synthetic", "config": {"workload": workload_desc(args.workload, cfg), "M": M, "N": N, "K": K,
                                        "parallelism": "rank 0 only"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                         "sample": "per step: X %d rows x W %d rows of the workload (K=%d), quantize + exact GEMM"
                                   % (rows[0], rows[1], K)},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "note": "the CPU oracle timed as it stands; no reference implementation exists for this hardware",
    }
    print(json.dumps(line))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="large")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank, local_rank, world = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, local_rank, world)


if __name__ == "__main__":
    main()
