"""Benchmark of the dynamic-FP8 hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload large|large4096|large8192|decode1|decode16|decode128|sweep|stack|backward|blockq|moe|...]

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
# layer: the large a8w8 layer, X and W quantized every step (default).
# decode: the same layer at small M; W quantized once before timing (weights
#   are static at inference), the step is quantize X + GEMM.
# sweep: quantize only, bf16 [8192, 8192]; every granularity x format.
# blockwise: block-wise quantize of the sweep input along its rows (E4M3 at
#   blocks of 128 and 32, stochastic E5M2 at 128) and the bf16 dequantize.
# blockscaled, blockscaled32: the large layer with block-wise scales along K
#   (E4M3, blocks of 128 / 32): X and W quantized block-wise every step, then
#   the block-scaled GEMM; blockscaled_mid / blockscaled32_mid: M=4096,
#   N=8192 at blocks of 128 / 32 (the ncu captures).
# blockq / blockq_unfused: the large layer whose result leaves as block-wise
#   E4M3 codes with one f32 scale per 32 columns of a row: written by the
#   GEMM's epilogue, or by a block-wise quantize of the bf16 result;
#   blockq8192: the fused form at M=8192 (the ncu capture).
# moe / moe_bf16: per-token quantize of the routed tokens + grouped a8w8 GEMM
#   over 64 experts (W quantized once); the bf16 grouped GEMM alone.
WORKLOADS = {
    "large": dict(kind="layer", M=16384, N=28672, K=8192),
    "large4096": dict(kind="layer", M=4096, N=28672, K=8192),
    "large8192": dict(kind="layer", M=8192, N=28672, K=8192),
    "decode1": dict(kind="decode", M=1, N=28672, K=8192),
    "decode16": dict(kind="decode", M=16, N=28672, K=8192),
    "decode128": dict(kind="decode", M=128, N=28672, K=8192),
    "sweep": dict(kind="sweep", M=8192, N=0, K=8192),
    "stack": dict(kind="stack", M=2048, N=4096, K=1024, steps_cycle=200, ring=16, fused=True),
    "stack_unfused": dict(kind="stack", M=2048, N=4096, K=1024, steps_cycle=200, ring=16, fused=False),
    "backward": dict(kind="backward", M=16384, N=28672, K=8192, ring=16),
    "blockwise": dict(kind="blockwise", M=8192, N=0, K=8192),
    "blockscaled": dict(kind="blockscaled", M=16384, N=28672, K=8192, block=128),
    "blockscaled32": dict(kind="blockscaled", M=16384, N=28672, K=8192, block=32),
    "blockscaled_mid": dict(kind="blockscaled", M=4096, N=8192, K=8192, block=128),
    "blockscaled32_mid": dict(kind="blockscaled", M=4096, N=8192, K=8192, block=32),
    "blockq": dict(kind="blockq", M=16384, N=28672, K=8192, fused=True),
    "blockq_unfused": dict(kind="blockq", M=16384, N=28672, K=8192, fused=False),
    "blockq8192": dict(kind="blockq", M=8192, N=28672, K=8192, fused=True),
    "moe": dict(kind="moe", M=32768, N=1408, K=2048, E=64),
    "moe_bf16": dict(kind="moe_bf16", M=32768, N=1408, K=2048, E=64),
}


def workload_desc(name, cfg):
    k = cfg["kind"]
    if k in ("layer", "decode"):
        return ("%s a8w8 GEMM layer: X bf16 [%d,%d] ~N(0,1) per-token E4M3, W bf16 [%d,%d] ~N(0,0.02) "
                "per-output-channel E4M3%s, out bf16 [%d,%d] (caller-owned)" %
                ("large" if k == "layer" else "decode", cfg["M"], cfg["K"], cfg["N"], cfg["K"],
                 "" if k == "layer" else " (quantized once: static weights)", cfg["M"], cfg["N"]))
    if k == "backward":
        return ("backward of the large a8w8 layer: grad g bf16 [%d,%d] ~N(0,1e-3) quantized per tensor with a "
                "delayed ring into row-major and transposed codes; W bf16 [%d,%d] and X bf16 [%d,%d] re-quantized "
                "transposed with their forward multipliers; grad_bias = g summed over rows, bf16 [%d]; "
                "dX = g W [%d,%d], dW = g^T X [%d,%d] on the NT GEMM" %
                (cfg["M"], cfg["N"], cfg["N"], cfg["K"], cfg["M"], cfg["K"], cfg["N"], cfg["M"], cfg["K"], cfg["N"],
                 cfg["K"]))
    if k == "stack":
        return ("delayed-scaling linear stack: X_t bf16 [2048,1024] (std 0.5 -> 8 over 200 steps), W_up bf16 "
                "[4096,1024], W_down bf16 [1024,4096] ~N(0,0.02); per-tensor E4M3 with four amax-history rings "
                "(length 16); h = GEMM(q(X), q(W_up)), y = GEMM(q(h), q(W_down)); step replayed as a CUDA graph; "
                "%s" % ("q(X), q(W_up), q(W_down) in one batched launch, q(h) in the first GEMM's epilogue"
                        if cfg.get("fused") else "four separate delayed quantizes"))
    if k == "sweep":
        return ("quantize sweep: bf16 [%d,%d] ~N(0,1), 0.1%% x100 outliers, 0.1%% zeros, one zero row; "
                "per-tensor / per-token / per-channel x E4M3 / E5M2" % (cfg["M"], cfg["K"]))
    if k == "blockscaled":
        return ("block-scaled a8w8 layer: X bf16 [%d,%d] ~N(0,1), W bf16 [%d,%d] ~N(0,0.02), both quantized "
                "block-wise to E4M3 with one f32 scale per %d elements along K every step, then the block-scaled "
                "GEMM, out bf16 [%d,%d] (caller-owned)" % (cfg["M"], cfg["K"], cfg["N"], cfg["K"], cfg["block"],
                                                          cfg["M"], cfg["N"]))
    if k == "blockq":
        return ("large a8w8 layer with a block-wise FP8 result: X bf16 [%d,%d] ~N(0,1) per-token E4M3, W bf16 "
                "[%d,%d] ~N(0,0.02) per-output-channel E4M3, result E4M3 [%d,%d] with one f32 scale per 32 columns "
                "of a row, %s" % (cfg["M"], cfg["K"], cfg["N"], cfg["K"], cfg["M"], cfg["N"],
                                  "quantized in the GEMM's epilogue" if cfg["fused"] else
                                  "from a bf16 result and a block-wise quantize"))
    if k == "blockwise":
        return ("block-wise quantize: bf16 [%d,%d] ~N(0,1) with the sweep's outliers and zeros, scales per block "
                "along the rows: E4M3 blocks of 128 and 32, stochastic E5M2 blocks of 128, and the bf16 "
                "dequantize of the E4M3 block-128 codes" % (cfg["M"], cfg["K"]))
    return ("grouped MoE GEMM: %d experts, K=%d, N=%d, %d tokens by Zipf(1.1) counts (2 experts empty); %s" %
            (cfg["E"], cfg["K"], cfg["N"], cfg["M"],
             "per-token E4M3 X + per-expert per-channel E4M3 W, a8w8" if k == "moe" else "bf16 X and W, fp32 acc"))


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
def q_bytes(rows, cols, nscales, elem=2):
    """Algorithmic bytes of one quantize call: read x, write codes and scales."""
    return rows * cols * (elem + 1) + 4 * nscales


def build(args, cfg, rank, dev, stream, peaks):
    """Device inputs and the step's calls for one workload.  Returns a dict:
    calls [(label, fn, launches)], per_step (flops or bytes), unit, e2e
    (copies + step), h2d/d2h bytes, roofline(ms_by_label), config extras."""
    import torch
    import workloads as W
    import fp8_dynamic_quantization_amax_b200 as hq

    kind = cfg["kind"]
    M, N, K = cfg["M"], cfg["N"], cfg["K"]
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16

    def bf16_host(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).pin_memory()

    if kind in ("layer", "decode"):
        x_host = bf16_host(W.large_x(M, K, seed=rank)).view(M, K)
        w_host = bf16_host(W.large_w(N, K)).view(N, K)
        x, w = x_host.to(dev), w_host.to(dev)
        xq = torch.empty((M, K), dtype=torch.uint8, device=dev)
        wq = torch.empty((N, K), dtype=torch.uint8, device=dev)
        xs = torch.empty((M,), dtype=torch.float32, device=dev)
        ws = torch.empty((N,), dtype=torch.float32, device=dev)
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        out_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
        qx = ("quantize X", lambda: hq.hq_quantize_fp8(x, hq.E4M3, hq.PER_TOKEN, q=xq, scales=xs, stream=stream), 1)
        qw = ("quantize W", lambda: hq.hq_quantize_fp8(w, hq.E4M3, hq.PER_TOKEN, q=wq, scales=ws, stream=stream), 1)
        gm = ("gemm", lambda: hq.hq_gemm_a8w8(xq, wq, xs, ws, hq.E4M3, out=out, stream=stream), 1)
        if kind == "decode":
            qw[1]()  # static weights: quantized once
        calls = [qx, qw, gm] if kind == "layer" else [qx, gm]
        decode_graphs = []
        if kind == "decode":
            # A decode step is two short kernels: each call is captured once as
            # a CUDA graph and replayed, as a serving loop would, so the step
            # is not paced by the Python binding's per-call work.
            def on_current(label):
                # launched on the stream current at call time: the capture stream while capturing
                if label == "quantize X":
                    return lambda: hq.hq_quantize_fp8(x, hq.E4M3, hq.PER_TOKEN, q=xq, scales=xs,
                                                      stream=torch.cuda.current_stream(dev))
                return lambda: hq.hq_gemm_a8w8(xq, wq, xs, ws, hq.E4M3, out=out, stream=torch.cuda.current_stream(dev))

            for c in calls:
                c[1]()  # first calls outside capture: one-time attribute and occupancy set-up
            torch.cuda.synchronize()
            ref = out.clone()
            graphed = []
            for label, _, n in calls:
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr):
                    on_current(label)()
                decode_graphs.append(gr)
                graphed.append((label, gr.replay, n))
            out.zero_()
            for _, fn, _ in graphed:
                fn()
            torch.cuda.synchronize()
            if not torch.equal(out.view(torch.int16), ref.view(torch.int16)):
                raise RuntimeError("the captured decode step does not reproduce the eager one")
            calls = graphed

        def e2e():
            x.copy_(x_host, non_blocking=True)
            if kind == "layer":
                w.copy_(w_host, non_blocking=True)
            for c in calls:
                c[1]()
            out_host.copy_(out, non_blocking=True)

        e2e_pipelined = None
        if kind == "layer":
            # a second set of step inputs and outputs, for a double-buffered run
            sets = [(x, w, out), (torch.empty_like(x), torch.empty_like(w), torch.empty_like(out))]
            s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

            def e2e_pipelined(n, e0, e1):
                """n steps through the public API, double-buffered: step i+1's
                host-to-device copies (one copy stream) and step i-1's
                device-to-host copy (another) overlap step i's kernels.  Every
                step still copies its inputs in and its result out."""
                h2d_done = [torch.cuda.Event() for _ in range(2)]
                comp_done = [torch.cuda.Event() for _ in range(2)]
                d2h_done = [torch.cuda.Event() for _ in range(2)]
                s_in.wait_stream(stream)
                e0.record(s_in)
                for i in range(n):
                    b = i % 2
                    xb, wb, ob = sets[b]
                    if i >= 2:
                        s_in.wait_event(comp_done[b])  # the kernels of step i-2 are done with these inputs
                    with torch.cuda.stream(s_in):
                        xb.copy_(x_host, non_blocking=True)
                        wb.copy_(w_host, non_blocking=True)
                    h2d_done[b].record(s_in)
                    stream.wait_event(h2d_done[b])
                    if i >= 2:
                        stream.wait_event(d2h_done[b])  # step i-2's result has been read back
                    hq.hq_quantize_fp8(xb, hq.E4M3, hq.PER_TOKEN, q=xq, scales=xs, stream=stream)
                    hq.hq_quantize_fp8(wb, hq.E4M3, hq.PER_TOKEN, q=wq, scales=ws, stream=stream)
                    hq.hq_gemm_a8w8(xq, wq, xs, ws, hq.E4M3, out=ob, stream=stream)
                    comp_done[b].record(stream)
                    s_out.wait_event(comp_done[b])
                    with torch.cuda.stream(s_out):
                        out_host.copy_(ob, non_blocking=True)
                    d2h_done[b].record(s_out)
                stream.wait_stream(s_in)
                stream.wait_stream(s_out)
                e1.record(stream)

        flops = 2.0 * M * N * K
        h2d = (M * K + (N * K if kind == "layer" else 0)) * 2

        def roofline(ms):
            g = ms["gemm"]
            if kind == "layer":
                a = flops / (g / 1e3) / 1e12
                traffic = traffic_from_profile("gemm.cu", "gemm_a8w8_large_M16384_N28672_K8192.md") \
                    if args.workload == "large" else None
                rf = {"bound": "tensor", "achieved": round(a, 1), "peak": round(fp8_peak, 1), "unit": "TFLOP/s",
                      "frac": round(a / fp8_peak, 4), "traffic": traffic,
                      "kernel": "k_gemm2<fp8, %s CTA-pair tile> (tcgen05 cta_group::2 kind::f8f6f4)" %
                                ("256x512" if M >= 8192 and N % 512 == 0 else "256x256"),
                      "peak_source": "%s bf16 burst %.1f TFLOP/s x %.0f (nominal fp8/bf16 dense ratio)" %
                                     (peaks["_src"], peaks["bf16_tflops"], FP8_OVER_BF16)}
            else:
                byts = N * K + M * K + 2 * M * N + 4 * (M + N)
                a = byts / (g / 1e3) / 1e9
                traffic = traffic_from_profile("gemm.cu", "gemm_a8w8_decode_M16_N28672_K8192.md") \
                    if args.workload == "decode16" else None
                rf = {"bound": "hbm", "achieved": round(a, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                      "frac": round(a / peaks["hbm_gbs"], 4), "traffic": traffic,
                      "kernel": "k_gemm<fp8, small-M tiles> (tcgen05 kind::f8f6f4, weight stream)",
                      "algorithmic_bytes": byts, "peak_source": "%s copy" % peaks["_src"]}
            return rf

        def extras(ms):
            qd = {"x_per_token": {"ms": round(ms["quantize X"], 4)}}
            qd["x_per_token"]["GB/s"] = round(q_bytes(M, K, M) / (ms["quantize X"] / 1e3) / 1e9, 1)
            qd["x_per_token"]["frac_hbm"] = round(qd["x_per_token"]["GB/s"] / peaks["hbm_gbs"], 4)
            if kind == "layer":
                gb = q_bytes(N, K, N) / (ms["quantize W"] / 1e3) / 1e9
                qd["w_per_channel"] = {"ms": round(ms["quantize W"], 4), "GB/s": round(gb, 1),
                                       "frac_hbm": round(gb / peaks["hbm_gbs"], 4)}
            qd["bytes"] = "algorithmic: 2 B read + 1 B write per element + 4 B per scale"
            d = {"quantize": qd, "gemm_ms": round(ms["gemm"], 4)}
            if kind == "decode":
                d["launch"] = "each call replayed from a CUDA graph captured once (static W quantized once)"
            return d

        l2 = "inputs larger than L2 (W %d MB, X %d MB, out %d MB); no flush" % (N * K * 2 >> 20, M * K * 2 >> 20,
                                                                               M * N * 2 >> 20)
        return dict(calls=calls, per_step=flops, unit="TFLOP/s", e2e=e2e, e2e_pipelined=e2e_pipelined, h2d=h2d,
                    d2h=M * N * 2,
                    roofline=roofline, extras=extras, l2=l2, flush=None, graphs=decode_graphs,
                    tensors=dict(xq=xq, wq=wq, xs=xs, ws=ws))

    if kind == "blockq":
        x_host = bf16_host(W.large_x(M, K, seed=rank)).view(M, K)
        w_host = bf16_host(W.large_w(N, K)).view(N, K)
        x, w = x_host.to(dev), w_host.to(dev)
        xq = torch.empty((M, K), dtype=torch.uint8, device=dev)
        wq = torch.empty((N, K), dtype=torch.uint8, device=dev)
        xs = torch.empty((M,), dtype=torch.float32, device=dev)
        ws = torch.empty((N,), dtype=torch.float32, device=dev)
        hq8 = torch.empty((M, N), dtype=torch.uint8, device=dev)
        hs = torch.empty((M, N // 32), dtype=torch.float32, device=dev)
        q_host = torch.empty((M, N), dtype=torch.uint8).pin_memory()
        s_host = torch.empty((M, N // 32), dtype=torch.float32).pin_memory()
        lib, P, st = hq.lib, (lambda t: t.data_ptr()), stream.cuda_stream
        calls = [("quantize X", lambda: hq.hq_quantize_fp8(x, hq.E4M3, hq.PER_TOKEN, q=xq, scales=xs, stream=stream), 1),
                 ("quantize W", lambda: hq.hq_quantize_fp8(w, hq.E4M3, hq.PER_TOKEN, q=wq, scales=ws, stream=stream), 1)]
        if cfg["fused"]:
            calls.append(("gemm", lambda: hq.check(lib.hq_gemm_a8w8_blockq(
                P(xq), P(wq), hq.E4M3, P(xs), M, P(ws), N, None, M, N, K, P(hq8), hq.E4M3, 32, P(hs), st)), 1))
        else:
            h = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            calls.append(("gemm", lambda: hq.hq_gemm_a8w8(xq, wq, xs, ws, hq.E4M3, out=h, stream=stream), 1))
            calls.append(("quantize h", lambda: hq.check(lib.hq_quantize_fp8_blockwise(
                P(h), hq.BF16, M, N, hq.E4M3, 32, 0, 0, P(hq8), P(hs), None, st)), 1))

        def e2e():
            x.copy_(x_host, non_blocking=True)
            w.copy_(w_host, non_blocking=True)
            for c in calls:
                c[1]()
            q_host.copy_(hq8, non_blocking=True)
            s_host.copy_(hs, non_blocking=True)

        flops = 2.0 * M * N * K

        def roofline(ms):
            t = ms["gemm"] + ms.get("quantize h", 0.0)
            a = flops / (t / 1e3) / 1e12
            return {"bound": "tensor", "achieved": round(a, 1), "peak": round(fp8_peak, 1), "unit": "TFLOP/s",
                    "frac": round(a / fp8_peak, 4), "traffic": None,
                    "kernel": ("k_gemm2<fp8, 256x512 CTA-pair tile> with the block-wise FP8 epilogue" if cfg["fused"]
                               else "k_gemm2<fp8, 256x512 CTA-pair tile> + the block-wise quantize of its bf16 result"),
                    "peak_source": "%s bf16 burst %.1f TFLOP/s x %.0f (nominal fp8/bf16 dense ratio)" %
                                   (peaks["_src"], peaks["bf16_tflops"], FP8_OVER_BF16)}

        def extras(ms):
            d = {"gemm_ms": round(ms["gemm"], 4), "result": "E4M3 [M, N] + f32 scales [M, N/32]"}
            if "quantize h" in ms:
                d["quantize_h_ms"] = round(ms["quantize h"], 4)
            return d

        l2 = "inputs larger than L2 (W %d MB, X %d MB, codes %d MB); no flush" % (N * K * 2 >> 20, M * K * 2 >> 20,
                                                                                 M * N >> 20)
        return dict(calls=calls, per_step=flops, unit="TFLOP/s", e2e=e2e, h2d=(M * K + N * K) * 2,
                    d2h=M * N + M * (N // 32) * 4, roofline=roofline, extras=extras, l2=l2, flush=None)

    if kind == "blockscaled":
        blk = cfg["block"]
        nb = -(-K // blk)
        x_host = bf16_host(W.large_x(M, K, seed=rank)).view(M, K)
        w_host = bf16_host(W.large_w(N, K)).view(N, K)
        x, w = x_host.to(dev), w_host.to(dev)
        xq = torch.empty((M, K), dtype=torch.uint8, device=dev)
        wq = torch.empty((N, K), dtype=torch.uint8, device=dev)
        xs = torch.empty((M, nb), dtype=torch.float32, device=dev)
        ws = torch.empty((N, nb), dtype=torch.float32, device=dev)
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        out_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
        lib, P, st = hq.lib, (lambda t: t.data_ptr()), stream.cuda_stream

        def qb(src, q, sc):
            rows, cols = src.shape
            hq.check(lib.hq_quantize_fp8_blockwise(P(src), hq.BF16, rows, cols, hq.E4M3, blk, 0, 0, P(q), P(sc),
                                                   None, st))

        calls = [("quantize X", lambda: qb(x, xq, xs), 1), ("quantize W", lambda: qb(w, wq, ws), 1),
                 ("gemm", lambda: hq.check(lib.hq_gemm_blockscaled(P(xq), P(wq), hq.E4M3, P(xs), P(ws), blk, None,
                                                                   M, N, K, P(out), st)), 1)]

        def e2e():
            x.copy_(x_host, non_blocking=True)
            w.copy_(w_host, non_blocking=True)
            for c in calls:
                c[1]()
            out_host.copy_(out, non_blocking=True)

        flops = 2.0 * M * N * K

        def roofline(ms):
            a = flops / (ms["gemm"] / 1e3) / 1e12
            return {"bound": "tensor", "achieved": round(a, 1), "peak": round(fp8_peak, 1), "unit": "TFLOP/s",
                    "frac": round(a / fp8_peak, 4), "traffic": None,
                    "kernel": "k_gemm_bs (tcgen05 kind::f8f6f4 per scale block, f32x2 promotion from TMEM)",
                    "peak_source": "%s bf16 burst %.1f TFLOP/s x %.0f (nominal fp8/bf16 dense ratio)" %
                                   (peaks["_src"], peaks["bf16_tflops"], FP8_OVER_BF16)}

        def extras(ms):
            d = {}
            for label, rows in (("quantize X", M), ("quantize W", N)):
                gb = q_bytes(rows, K, rows * nb) / (ms[label] / 1e3) / 1e9
                d[label] = {"ms": round(ms[label], 4), "GB/s": round(gb, 1), "frac_hbm": round(gb / peaks["hbm_gbs"], 4)}
            return {"quantize_blockwise": d, "gemm_ms": round(ms["gemm"], 4), "block": blk}

        l2 = "inputs larger than L2 (W %d MB, X %d MB, out %d MB); no flush" % (N * K * 2 >> 20, M * K * 2 >> 20,
                                                                               M * N * 2 >> 20)
        return dict(calls=calls, per_step=flops, unit="TFLOP/s", e2e=e2e, h2d=(M * K + N * K) * 2, d2h=M * N * 2,
                    roofline=roofline, extras=extras, l2=l2, flush=None)

    if kind == "backward":
        Lr = cfg["ring"]
        g_host = bf16_host(W.f32_to_bf16_bits(W.normal((M, N), 1e-3, 100 + rank))).view(M, N)
        x_host = bf16_host(W.large_x(M, K, seed=rank)).view(M, K)
        w_dev = bf16_host(W.large_w(N, K)).view(N, K).to(dev)
        g, x = g_host.to(dev), x_host.to(dev)
        ring = torch.zeros(Lr + 2, dtype=torch.float32, device=dev)
        ring[Lr] = 448.0 / 4e-3  # E4M3 max over an expected gradient amax
        # the forward's multipliers of W and X (their dynamic per-tensor scales)
        _, sw0 = hq.hq_quantize_fp8(w_dev, hq.E4M3, hq.PER_TENSOR)
        _, sx0 = hq.hq_quantize_fp8(x, hq.E4M3, hq.PER_TENSOR)
        mw, mx = 1.0 / sw0, 1.0 / sx0
        g8 = torch.empty((M, N), dtype=torch.uint8, device=dev)
        gT8 = torch.empty((N, M), dtype=torch.uint8, device=dev)
        wT8 = torch.empty((K, N), dtype=torch.uint8, device=dev)
        xT8 = torch.empty((K, M), dtype=torch.uint8, device=dev)
        sg, sw, sx = (torch.empty((1,), dtype=torch.float32, device=dev) for _ in range(3))
        dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
        dW = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
        db = torch.empty((N,), dtype=torch.bfloat16, device=dev)
        dX_host = torch.empty((M, K), dtype=torch.bfloat16).pin_memory()
        dW_host = torch.empty((N, K), dtype=torch.bfloat16).pin_memory()
        db_host = torch.empty((N,), dtype=torch.bfloat16).pin_memory()
        wsg, wsw, wsx = (torch.zeros(256, dtype=torch.uint8, device=dev) for _ in range(3))
        wsb = torch.zeros(hq.hq_grad_bias_workspace_bytes(M, N), dtype=torch.uint8, device=dev)
        lib, P = hq.lib, (lambda t: None if t is None else t.data_ptr())
        st = stream.cuda_stream
        counter = [0]

        def qt(src, qo, qt_, scale, mult=None, rg=None, idx=0, ws_=None):
            rows, cols = src.shape
            hq.check(lib.hq_quantize_fp8_transpose(P(src), hq.BF16, rows, cols, hq.E4M3, P(qo), P(qt_), P(scale),
                                                   None, P(mult), P(rg), Lr if rg is not None else 0, idx, 0,
                                                   P(ws_), ws_.numel(), st))

        def quant():
            qt(g, g8, gT8, sg, rg=ring, idx=counter[0] % Lr, ws_=wsg)
            counter[0] += 1
            qt(w_dev, None, wT8, sw, mult=mw, ws_=wsw)
            qt(x, None, xT8, sx, mult=mx, ws_=wsx)

        def gemms():
            hq.hq_gemm_a8w8(g8, wT8, sg, sw, hq.E4M3, out=dX, stream=stream)
            hq.hq_gemm_a8w8(gT8, xT8, sg, sx, hq.E4M3, out=dW, stream=stream)

        def grad_bias():
            hq.check(lib.hq_grad_bias(P(g), hq.BF16, M, N, P(db), P(wsb), wsb.numel(), st))

        calls = [("quantize g, W^T, X^T", quant, 3), ("grad_bias", grad_bias, 1), ("dX and dW GEMMs", gemms, 2)]

        def e2e():
            g.copy_(g_host, non_blocking=True)
            x.copy_(x_host, non_blocking=True)
            quant()
            grad_bias()
            gemms()
            dX_host.copy_(dX, non_blocking=True)
            dW_host.copy_(dW, non_blocking=True)
            db_host.copy_(db, non_blocking=True)

        flops = 2.0 * 2 * M * N * K

        def roofline(ms):
            a = flops / (ms["dX and dW GEMMs"] / 1e3) / 1e12
            return {"bound": "tensor", "achieved": round(a, 1), "peak": round(fp8_peak, 1), "unit": "TFLOP/s",
                    "frac": round(a / fp8_peak, 4), "traffic": None,
                    "kernel": "k_gemm2<fp8, 256x512 CTA-pair tile> (dX and dW)",
                    "peak_source": "%s bf16 burst x 2 (nominal fp8/bf16)" % peaks["_src"]}

        def extras(ms):
            qbytes = (M * N * 2 + 2 * M * N) + (N * K * 2 + N * K) + (M * K * 2 + M * K)
            gb = qbytes / (ms["quantize g, W^T, X^T"] / 1e3) / 1e9
            bb = (M * N * 2 + N * 2) / (ms["grad_bias"] / 1e3) / 1e9
            return {"quantize_transpose": {"ms": round(ms["quantize g, W^T, X^T"], 4), "GB/s": round(gb, 1),
                                           "frac_hbm": round(gb / peaks["hbm_gbs"], 4),
                                           "bytes": "g: 2 B read + 2 x 1 B codes; W, X: 2 B read + 1 B codes"},
                    "grad_bias": {"ms": round(ms["grad_bias"], 4), "GB/s": round(bb, 1),
                                  "frac_hbm": round(bb / peaks["hbm_gbs"], 4),
                                  "bytes": "g: 2 B read per element + 2 B per column"},
                    "gemm_ms": round(ms["dX and dW GEMMs"], 4)}

        return dict(calls=calls, per_step=flops, unit="TFLOP/s", e2e=e2e, h2d=(M * N + M * K) * 2,
                    d2h=(M * K + N * K + N) * 2, roofline=roofline, extras=extras, flush=None,
                    l2="inputs larger than L2 (g %d MB, X %d MB, W %d MB); no flush" %
                       (M * N * 2 >> 20, M * K * 2 >> 20, N * K * 2 >> 20))

    if kind == "stack":
        T, D, H, L = M, K, N, cfg["ring"]
        cyc = cfg["steps_cycle"]
        xs_host = [bf16_host(W.delayed_x(t, T, D, cyc)).view(T, D) for t in range(cyc)]
        xs_dev = torch.stack([x.to(dev) for x in xs_host])
        wu = bf16_host(W.f32_to_bf16_bits(W.normal((H, D), 0.02, 1))).view(H, D).to(dev)
        wd = bf16_host(W.f32_to_bf16_bits(W.normal((D, H), 0.02, 2))).view(D, H).to(dev)
        rings = {k: torch.zeros(L + 2, dtype=torch.float32, device=dev) for k in ("x", "wu", "h", "wd")}
        for r in rings.values():
            r[L] = 1.0
        def u8(r, c):
            return torch.empty((r, c), dtype=torch.uint8, device=dev)
        def f1():
            return torch.empty((1,), dtype=torch.float32, device=dev)
        pipe = cfg["fused"]
        nb = 2 if pipe else 1  # code / scale buffers of X, W_up, W_down: one per step parity when pipelined
        xq, wuq, wdq = [u8(T, D) for _ in range(nb)], [u8(H, D) for _ in range(nb)], [u8(D, H) for _ in range(nb)]
        xsc, wusc, wdsc = [f1() for _ in range(nb)], [f1() for _ in range(nb)], [f1() for _ in range(nb)]
        hq_, hsc = u8(T, H), f1()
        h = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        y = torch.empty((T, D), dtype=torch.bfloat16, device=dev)
        y_host = torch.empty((T, D), dtype=torch.bfloat16).pin_memory()
        ws = {k: torch.zeros(hq.hq_quantize_workspace_bytes(hq.PER_TENSOR, 1, 1, True), dtype=torch.uint8, device=dev)
              for k in rings}
        side = torch.cuda.Stream(dev) if pipe else None
        assert cyc % 2 == 0  # buffer parity stays aligned with the step index across the cycle

        def quantize_batch(t, b, st):
            # X_t (resident), W_up and W_down with their rings, slot t mod L, in one launch
            idx = t % L
            hq.hq_quantize_fp8_delayed_batch(
                [dict(x=xs_dev[t], ring=rings["x"], ring_idx=idx, q=xq[b], scale=xsc[b], workspace=ws["x"]),
                 dict(x=wu, ring=rings["wu"], ring_idx=idx, q=wuq[b], scale=wusc[b], workspace=ws["wu"]),
                 dict(x=wd, ring=rings["wd"], ring_idx=idx, q=wdq[b], scale=wdsc[b], workspace=ws["wd"])],
                hq.E4M3, stream=st)

        def body(t):
            st = torch.cuda.current_stream(dev)
            idx = t % L
            if pipe:
                # step t's two GEMMs read the codes that step t-1 quantized into
                # buffer t mod 2; step t+1's batched quantize writes the other
                # buffer on a side stream beside the second GEMM, whose 128
                # tiles leave 20 SMs free (each ring still sees its updates
                # in step order).  h leaves the first GEMM as FP8 codes, its
                # delayed quantize (ring h) run by the epilogue.
                b = t % 2
                hq.hq_gemm_a8w8_ex(xq[b], wuq[b], xsc[b], wusc[b], hq.E4M3, q_out=hq_, q_fmt=hq.E4M3, q_scale=hsc,
                                   ring=rings["h"], ring_idx=idx, workspace=ws["h"], stream=st)
                side.wait_stream(st)
                hq.hq_gemm_a8w8(hq_, wdq[b], hsc, wdsc[b], hq.E4M3, out=y, stream=st)
                with torch.cuda.stream(side):
                    quantize_batch((t + 1) % cyc, 1 - b, side)
                st.wait_stream(side)
                return

            def q(x, key, qo, so):
                hq.hq_quantize_fp8(x, hq.E4M3, hq.PER_TENSOR, q=qo, scales=so, ring=rings[key], ring_idx=idx,
                                   workspace=ws[key], stream=st)
            q(xs_dev[t], "x", xq[0], xsc[0])
            q(wu, "wu", wuq[0], wusc[0])
            hq.hq_gemm_a8w8(xq[0], wuq[0], xsc[0], wusc[0], hq.E4M3, out=h, stream=st)
            q(h, "h", hq_, hsc)
            q(wd, "wd", wdq[0], wdsc[0])
            hq.hq_gemm_a8w8(hq_, wdq[0], hsc, wdsc[0], hq.E4M3, out=y, stream=st)

        def reset():
            # fresh rings; when pipelined, step 0's quantize runs here, ahead of step 0
            for r in rings.values():
                r.zero_()
                r[L] = 1.0
            if pipe:
                quantize_batch(0, 0, torch.cuda.current_stream(dev))

        # one graph per step of the cycle: X_t's address, the ring slot and
        # the buffer parity are launch arguments, so no input copy is needed
        reset()
        for t in range(L):
            body(t)
        torch.cuda.synchronize()
        graph_error = None
        graphs = []
        try:
            for t in range(cyc):
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr):
                    body(t)
                graphs.append(gr)
        except Exception as exc:  # eager launches instead; the line says so
            graphs = None
            graph_error = "%s: %s" % (type(exc).__name__, str(exc).splitlines()[0] if str(exc) else "")
            torch.cuda.synchronize()
        reset()  # the warm-up and capture passes ran the rings: start fresh
        counter = [0]

        def step_fn():
            t = counter[0] % cyc
            counter[0] += 1
            if graphs is not None:
                graphs[t].replay()
            else:
                body(t)

        def e2e():
            t = counter[0] % cyc
            counter[0] += 1
            tin = (t + 1) % cyc if pipe else t  # the X this step's quantize reads
            xs_dev[tin].copy_(xs_host[tin], non_blocking=True)
            if graphs is not None:
                graphs[t].replay()
            else:
                body(t)
            y_host.copy_(y, non_blocking=True)

        flops = 2.0 * T * H * D * 2

        def roofline(ms):
            a = flops / (ms["step"] / 1e3) / 1e12
            return {"bound": "tensor", "achieved": round(a, 1), "peak": round(fp8_peak, 1), "unit": "TFLOP/s",
                    "frac": round(a / fp8_peak, 4), "traffic": None,
                    "kernel": "the whole step (2 GEMMs + 4 delayed quantizes) as one CUDA graph replay",
                    "peak_source": "%s bf16 burst x 2 (nominal fp8/bf16)" % peaks["_src"]}

        def extras(ms):
            d = {"kernels_per_step": 3 if cfg["fused"] else 6,
                 "rings": "4 x [16 hist | scale | counter], updated on the device every step",
                 "quantize": ("X, W_up, W_down in one batched launch; h in the first GEMM's epilogue; step t+1's "
                              "batched quantize runs on a second stream inside step t's graph, beside step t's "
                              "GEMMs (codes and scales double-buffered by step parity)"
                              if cfg["fused"] else "four separate delayed quantizes (h from a bf16 round trip)")}
            if graphs is not None:
                d["graph_launches_per_step"] = 1
            else:
                d["graph_capture"] = "failed (%s); eager launches" % graph_error
            return d

        return dict(calls=[("step", step_fn, 3 if cfg["fused"] else 6)], per_step=flops, unit="TFLOP/s", e2e=e2e,
                    h2d=T * D * 2,
                    d2h=T * D * 2, roofline=roofline, extras=extras, flush=None, graphs=graphs,
                    tensors=dict(y=y, rings=rings),
                    l2="working set (X 4 MB, W 16 MB, h 16 MB) fits L2: a steady-state layer step")

    if kind == "sweep":
        x_host = bf16_host(W.sweep(M, K, seed=rank)).view(M, K)
        x = x_host.to(dev)
        flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev).fill_(1)
        sink = torch.empty((), dtype=torch.uint8, device=dev)
        calls, outs, per = [], [], 0
        names = {hq.PER_TENSOR: "tensor", hq.PER_TOKEN: "token", hq.PER_CHANNEL: "channel"}
        for fmt in (hq.E4M3, hq.E5M2):
            for g in (hq.PER_TENSOR, hq.PER_TOKEN, hq.PER_CHANNEL):
                ns = hq.hq_scale_count(g, M, K)
                q = torch.empty((M, K), dtype=torch.uint8, device=dev)
                sc = torch.empty((ns,), dtype=torch.float32, device=dev)
                outs.append((q, sc, torch.empty((M, K), dtype=torch.uint8).pin_memory(),
                             torch.empty((ns,), dtype=torch.float32).pin_memory()))
                launches = 1  # at this size every mode is one launch (per-tensor / per-channel: cooperative)
                calls.append(("%s %s" % (names[g], "e4m3" if fmt == hq.E4M3 else "e5m2"),
                              (lambda g=g, fmt=fmt, q=q, sc=sc:
                               hq.hq_quantize_fp8(x, fmt, g, q=q, scales=sc, stream=stream)), launches))
                per += q_bytes(M, K, ns)

        def e2e():
            x.copy_(x_host, non_blocking=True)
            for c, (q, sc, qh, sh) in zip(calls, outs):
                c[1]()
                qh.copy_(q, non_blocking=True)
                sh.copy_(sc, non_blocking=True)

        def roofline(ms):
            label = max(ms, key=ms.get)
            ns = {"tensor": 1, "token": M, "channel": K}[label.split()[0]]
            a = q_bytes(M, K, ns) / (ms[label] / 1e3) / 1e9
            return {"bound": "hbm", "achieved": round(a, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": round(a / peaks["hbm_gbs"], 4), "traffic": None,
                    "kernel": "quantize %s (the slowest mode)" % label, "peak_source": "%s copy" % peaks["_src"]}

        def extras(ms):
            d = {}
            for label, t in ms.items():
                ns = {"tensor": 1, "token": M, "channel": K}[label.split()[0]]
                gb = q_bytes(M, K, ns) / (t / 1e3) / 1e9
                d[label] = {"ms": round(t, 4), "GB/s": round(gb, 1), "frac_hbm": round(gb / peaks["hbm_gbs"], 4)}
            return {"quantize": d}

        return dict(calls=calls, per_step=per, unit="GB/s", e2e=e2e, h2d=M * K * 2,
                    d2h=sum(q.numel() + 4 * sc.numel() for q, sc, _, _ in outs), roofline=roofline,
                    extras=extras, flush=lambda: torch.amax(flush, dim=0, out=sink),
                    l2="L2 flushed (512 MB read) before every call; value = bytes / summed call times")

    if kind == "blockwise":
        x_host = bf16_host(W.sweep(M, K, seed=rank)).view(M, K)
        x = x_host.to(dev)
        flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev).fill_(1)
        sink = torch.empty((), dtype=torch.uint8, device=dev)
        lib, P, st = hq.lib, (lambda t: t.data_ptr()), stream.cuda_stream
        modes = [("e4m3 b128", hq.E4M3, 128, 0), ("e4m3 b32", hq.E4M3, 32, 0), ("e5m2 sr b128", hq.E5M2, 128, 1)]
        calls, outs, per, bytes_of = [], [], 0, {}
        for label, fmt, blk, sr in modes:
            q = torch.empty((M, K), dtype=torch.uint8, device=dev)
            sc = torch.empty((M, -(-K // blk)), dtype=torch.float32, device=dev)
            outs.append((q, sc, torch.empty((M, K), dtype=torch.uint8).pin_memory(),
                         torch.empty(tuple(sc.shape), dtype=torch.float32).pin_memory()))
            calls.append(("quantize " + label,
                          (lambda fmt=fmt, blk=blk, sr=sr, q=q, sc=sc:
                           hq.check(lib.hq_quantize_fp8_blockwise(P(x), hq.BF16, M, K, fmt, blk, sr, 2024, P(q),
                                                                  P(sc), None, st))), 1))
            bytes_of["quantize " + label] = q_bytes(M, K, sc.numel())
        q128, s128 = outs[0][0], outs[0][1]
        deq = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
        deq_host = torch.empty((M, K), dtype=torch.bfloat16).pin_memory()
        calls.append(("dequantize e4m3 b128 -> bf16",
                      lambda: hq.check(lib.hq_dequantize_fp8_blockwise(P(q128), hq.E4M3, M, K, 128, P(s128), hq.BF16,
                                                                       P(deq), st)), 1))
        bytes_of["dequantize e4m3 b128 -> bf16"] = M * K * 3 + 4 * s128.numel()
        per = sum(bytes_of.values())

        def e2e():
            x.copy_(x_host, non_blocking=True)
            for c, (q, sc, qh, sh) in zip(calls, outs):
                c[1]()
                qh.copy_(q, non_blocking=True)
                sh.copy_(sc, non_blocking=True)
            calls[-1][1]()
            deq_host.copy_(deq, non_blocking=True)

        def roofline(ms):
            label = "quantize e4m3 b128"
            a = bytes_of[label] / (ms[label] / 1e3) / 1e9
            return {"bound": "hbm", "achieved": round(a, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": round(a / peaks["hbm_gbs"], 4), "traffic": None,
                    "kernel": "k_block_tma_narrow (E4M3, blocks of 128)", "peak_source": "%s copy" % peaks["_src"]}

        def extras(ms):
            d = {}
            for label, t in ms.items():
                gb = bytes_of[label] / (t / 1e3) / 1e9
                d[label] = {"ms": round(t, 4), "GB/s": round(gb, 1), "frac_hbm": round(gb / peaks["hbm_gbs"], 4)}
            return {"blockwise": d}

        return dict(calls=calls, per_step=per, unit="GB/s", e2e=e2e, h2d=M * K * 2,
                    d2h=sum(q.numel() + 4 * sc.numel() for q, sc, _, _ in outs) + M * K * 2, roofline=roofline,
                    extras=extras, flush=lambda: torch.amax(flush, dim=0, out=sink),
                    l2="L2 flushed (512 MB read) before every call; value = bytes / summed call times")

    # moe / moe_bf16
    E = cfg["E"]
    xb, wb, off = W.moe_inputs(E, M, N, K, seed=rank)
    x_host = bf16_host(xb).view(M, K)
    w_host = bf16_host(wb).view(E, N, K)
    x, w = x_host.to(dev), w_host.to(dev)
    offd = torch.from_numpy(off).to(dev)
    out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    out_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    flops = 2.0 * M * N * K
    if kind == "moe":
        xq = torch.empty((M, K), dtype=torch.uint8, device=dev)
        xs = torch.empty((M,), dtype=torch.float32, device=dev)
        wq, ws = hq.hq_quantize_fp8(w.view(E * N, K), hq.E4M3, hq.PER_TOKEN, stream=stream)  # static weights
        wq = wq.view(E, N, K)
        calls = [("quantize X", lambda: hq.hq_quantize_fp8(x, hq.E4M3, hq.PER_TOKEN, q=xq, scales=xs, stream=stream), 1),
                 ("gemm", lambda: hq.hq_grouped_gemm_a8w8(xq, wq, xs, ws, offd, out=out, stream=stream), 1)]
        peak, dt = fp8_peak, "fp8"
    else:
        calls = [("gemm", lambda: hq.hq_grouped_gemm_bf16(x, w, offd, out=out, stream=stream), 1)]
        peak, dt = peaks["bf16_tflops"], "bf16"

    def e2e():
        x.copy_(x_host, non_blocking=True)
        for c in calls:
            c[1]()
        out_host.copy_(out, non_blocking=True)

    def roofline(ms):
        a = flops / (ms["gemm"] / 1e3) / 1e12
        return {"bound": "tensor", "achieved": round(a, 1), "peak": round(peak, 1), "unit": "TFLOP/s",
                "frac": round(a / peak, 4), "traffic": None,
                "kernel": "k_gemm2<%s, grouped 256x256 CTA-pair tiles> (tcgen05 cta_group::2)" % dt,
                "peak_source": "%s bf16 burst%s" % (peaks["_src"], " x 2 (nominal fp8/bf16)" if dt == "fp8" else "")}

    def extras(ms):
        d = {"gemm_ms": round(ms["gemm"], 4)}
        if "quantize X" in ms:
            gb = q_bytes(M, K, M) / (ms["quantize X"] / 1e3) / 1e9
            d["quantize"] = {"x_per_token": {"ms": round(ms["quantize X"], 4), "GB/s": round(gb, 1),
                                             "frac_hbm": round(gb / peaks["hbm_gbs"], 4)}}
        return d

    return dict(calls=calls, per_step=flops, unit="TFLOP/s", e2e=e2e, h2d=M * K * 2, d2h=M * N * 2,
                roofline=roofline, extras=extras, flush=None,
                l2="inputs larger than L2 (X %d MB, W %d MB, out %d MB); no flush" %
                   (M * K * 2 >> 20, E * N * K * (1 if kind == "moe" else 2) >> 20, M * N * 2 >> 20))


def time_workload(wl, steps, warmup, stream, world, dev, hq):
    """Warm-up, then exactly `steps` steps bracketed by a barrier and a device
    synchronise, with CUDA events on the launching stream around every call
    and clocks sampled during the timed region.  Returns the per-call mean
    times, the timed region's milliseconds (max over ranks) and the clocks."""
    import torch
    import torch.distributed as dist

    calls = wl["calls"]

    def step(ev=None):
        for j, (_, fn, _) in enumerate(calls):
            if wl["flush"] is not None:
                wl["flush"]()
            if ev is not None:
                ev[2 * j].record(stream)
            fn()
            if ev is not None:
                ev[2 * j + 1].record(stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    hq.hq_check_device_error()

    clocks = ClockSampler(dev.index)
    clocks.start()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * len(calls))] for _ in range(steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    hq.hq_check_device_error()
    ms_by = {c[0]: statistics.mean(e[2 * j].elapsed_time(e[2 * j + 1]) for e in evs) for j, c in enumerate(calls)}
    region = t0.elapsed_time(t1)
    if wl["flush"] is not None:  # flushes sit between the calls: time the calls alone
        region = sum(sum(e[2 * j].elapsed_time(e[2 * j + 1]) for j in range(len(calls))) for e in evs)
    return ms_by, max_over_ranks(region, world, dev), clk


# Workloads measured beside the default one, in the same process, so that its
# line carries the whole metric: the quantize sweep, the grouped MoE GEMMs and
# the delayed-scaling stack step (steps per workload).
COMPANIONS = (("sweep", 10), ("moe", 20), ("moe_bf16", 20), ("stack", 200))


def companion_line(args, name, steps, rank, world, dev, stream, peaks, hq):
    import torch

    cfg = WORKLOADS[name]
    sub = argparse.Namespace(**dict(vars(args), workload=name))
    wl = build(sub, cfg, rank, dev, stream, peaks)
    ms_by, ms, clk = time_workload(wl, steps, 5, stream, world, dev, hq)
    scale = 1e12 if wl["unit"] == "TFLOP/s" else 1e9
    d = {"workload": workload_desc(name, cfg), "value": round(wl["per_step"] * steps * world / (ms / 1e3) / scale, 2),
         "unit": wl["unit"], "steps": steps, "warmup": 5, "ms_per_step": round(ms / steps, 4),
         "roofline": wl["roofline"](ms_by), "call_ms": {k: round(v, 4) for k, v in ms_by.items()},
         "l2": wl["l2"], "gpu_launches": sum(c[2] for c in wl["calls"]) * steps,
         "clocks": {"sm_mhz": clk.get("sm_mhz"), "reasons": clk.get("reasons")}}
    d.update(wl["extras"](ms_by))
    wl.pop("graphs", None)
    del wl
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return d


def scaled_mm_ceiling(t, M, N, K, stream, fp8_peak, reps=10):
    """torch._scaled_mm (a library FP8 GEMM with row-wise scales) on the same
    codes and scales, timed with CUDA events: a stated ceiling for the large
    layer's GEMM, not part of the measured path."""
    import torch

    try:
        a = t["xq"].view(torch.float8_e4m3fn)
        b = t["wq"].view(torch.float8_e4m3fn).t()  # [K, N], column-major
        sa, sb = t["xs"].view(M, 1), t["ws"].view(1, N)
        for _ in range(3):
            out = torch._scaled_mm(a, b, scale_a=sa, scale_b=sb, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            out = torch._scaled_mm(a, b, scale_a=sa, scale_b=sb, out_dtype=torch.bfloat16)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        del out
        tf = 2.0 * M * N * K / (ms / 1e3) / 1e12
        return {"op": "torch._scaled_mm, E4M3 row-wise scales, bf16 out (library GEMM; a ceiling, not a target)",
                "ms": round(ms, 4), "TFLOP/s": round(tf, 1), "frac_of_fp8_peak": round(tf / fp8_peak, 4),
                "reps": reps}
    except Exception as exc:  # the ceiling is context only: record why it is missing
        return {"op": "torch._scaled_mm", "unavailable": "%s: %s" % (type(exc).__name__, str(exc).splitlines()[0])}


def run_ours(args, rank, local_rank, world):
    import torch
    import torch.distributed as dist

    import fp8_dynamic_quantization_amax_b200 as hq

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    cfg = WORKLOADS[args.workload]
    peaks, peak_src = load_peaks()
    peaks = dict(peaks, _src=peak_src)
    stream = torch.cuda.current_stream(dev)
    wl = build(args, cfg, rank, dev, stream, peaks)
    calls = wl["calls"]
    ms_by, ms, clk = time_workload(wl, args.steps, args.warmup, stream, world, dev, hq)
    scale = 1e12 if wl["unit"] == "TFLOP/s" else 1e9
    value = wl["per_step"] * args.steps * world / (ms / 1e3) / scale

    # end to end through the C ABI with host buffers: the step's H2D copies,
    # its kernels and the D2H of its results, every step (double-buffered
    # across steps where the workload provides it)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    pipelined = wl.get("e2e_pipelined")
    if pipelined is not None:
        e2e_steps = max(1, min(args.steps, 8))
        pipelined(2, e0, e1)  # warm-up
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        pipelined(e2e_steps, e0, e1)
    else:
        e2e_steps = max(1, min(args.steps, 5))
        wl["e2e"]()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0.record(stream)
        for _ in range(e2e_steps):
            wl["e2e"]()
        e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = wl["per_step"] * e2e_steps * world / (e2e_ms / 1e3) / scale

    # the default workload's line also carries the rest of the metric
    also = None
    if args.workload == "large" and not args.no_companions:
        fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
        also = {"scaled_mm_ceiling": scaled_mm_ceiling(wl["tensors"], cfg["M"], cfg["N"], cfg["K"], stream,
                                                       fp8_peak)}
        for name, steps in COMPANIONS:
            also[name] = companion_line(args, name, steps, rank, world, dev, stream, peaks, hq)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and cfg["kind"] in ("layer", "decode"):
        mx = min(256, cfg["M"])
        cpu = cpu_baseline(cfg["M"], cfg["N"], cfg["K"], budget_rows=(mx, min(cfg["N"], 4096 * 256 // mx)))
    elif rank == 0 and world == 1 and not args.no_cpu_baseline and cfg["kind"] == "blockscaled":
        mx, nw = 256, 4096
        fl, dt = cpu_blockscaled_sample(cfg["M"], cfg["N"], cfg["K"], cfg["block"], (mx, nw))
        cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
               "sample": "X %d rows x W %d rows (K=%d, block %d): block-wise quantize of both + exact block-scaled "
                         "GEMM, %.1f s" % (mx, nw, cfg["K"], cfg["block"], dt), "seconds": round(dt, 2)}
    elif rank == 0 and world == 1 and not args.no_cpu_baseline and cfg["kind"] in ("sweep", "blockwise"):
        rows = 256
        fn = cpu_sweep_sample if cfg["kind"] == "sweep" else cpu_blockwise_sample
        byts, dt = fn(rows, cfg["K"])
        cpu = {"value": byts / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
               "sample": "%d rows x %d cols of the workload's input, every call of the step, %.1f s"
                         % (rows, cfg["K"], dt), "seconds": round(dt, 2)}
    if cpu is not None:
        cpu["host"] = host_cpu()

    wl.pop("graphs", None)  # release captured graphs before the process group goes
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": wl["unit"],
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": ("bf16 -> fp8 codes + f32 scales" if cfg["kind"] in ("sweep", "blockwise") else
                  "fp8_e4m3 (fp32 accumulate, block-wise E4M3 out)" if cfg["kind"] == "blockq" else
                  "fp8_e4m3 (fp32 accumulate, bf16 out)" if cfg["kind"] != "moe_bf16" else "bf16 (fp32 accumulate)"),
        "data": "synthetic (seeded host generators; X seed = rank)",
        "config": {"workload": workload_desc(args.workload, cfg), "M": cfg["M"], "N": cfg["N"], "K": cfg["K"],
                   "l2": wl["l2"], "parallelism": "dp%d" % world},
        "roofline": wl["roofline"](ms_by),
        "call_ms": {k: round(v, 4) for k, v in ms_by.items()},
        "clocks": clk,
        "e2e": dict({"value": round(e2e_value, 2), "unit": wl["unit"], "h2d_bytes_per_step": wl["h2d"],
                     "d2h_bytes_per_step": wl["d2h"], "steps": e2e_steps},
                    **({"pipelined": "double-buffered: step i+1's host-to-device copies and step i-1's "
                                     "device-to-host copy run on two copy streams while step i's kernels run; "
                                     "the timed region spans the first copy in to the last copy out"}
                       if pipelined is not None else {})),
        "gpu_launches": sum(c[2] for c in calls) * args.steps,
        "cpu_baseline": cpu,
    }
    line.update(wl["extras"](ms_by))
    if also is not None:
        line["also"] = also
    print(json.dumps(line))


def host_cpu():
    """The host's logical CPU count, the CPUs this process may use, and the
    CPU model name."""
    model = None
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                model = ln.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    try:
        usable = len(os.sched_getaffinity(0))
    except AttributeError:
        usable = os.cpu_count()
    return {"nproc": os.cpu_count(), "usable": usable, "model": model}


# --------------------------------------------------------------- oracle
def cpu_baseline(M, N, K, budget_rows, seed=0, all_cores=True):
    """The oracle, as it stands, on a bounded sample of the workload: per-token
    quantize of `mx` rows of X and `nw` rows of W, then the exact GEMM of the
    sample.  Returns TFLOP/s of the sample's GEMM flops per oracle time: on
    one core, and (all_cores) on every usable core, each thread running the
    unchanged single-threaded oracle on its own slice of rows."""
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
    d = {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
         "sample": "X %d rows x W %d rows (K=%d): per-token quantize of both + exact GEMM, %.1f s"
                   % (mx, nw, K, dt),
         "seconds": round(dt, 2)}
    if not all_cores:
        return d
    import concurrent.futures as cf
    try:
        threads = len(os.sched_getaffinity(0))
    except AttributeError:
        threads = os.cpu_count() or 1

    def slices(n):
        step = -(-n // threads)
        return [(i, min(n, i + step)) for i in range(0, n, step)]

    t = time.perf_counter()
    with cf.ThreadPoolExecutor(threads) as ex:  # the oracle's C calls release the GIL
        xp = list(ex.map(lambda r: O.quantize(x[r[0]:r[1]], O.E4M3, O.PER_TOKEN), slices(mx)))
        wp = list(ex.map(lambda r: O.quantize(w[r[0]:r[1]], O.E4M3, O.PER_TOKEN), slices(nw)))
        xq2, xs2 = np.concatenate([p[0] for p in xp]), np.concatenate([p[1] for p in xp])
        wq2, ws2 = np.concatenate([p[0] for p in wp]), np.concatenate([p[1] for p in wp])
        list(ex.map(lambda r: O.gemm_a8w8(xq2[r[0]:r[1]], wq2, O.E4M3, xs2[r[0]:r[1]], ws2), slices(mx)))
    dta = time.perf_counter() - t
    single = dict(d)
    d.update({"value": flops / dta / 1e12, "cores": threads, "seconds": round(dta, 2),
              "sample": "the same sample on %d threads (each runs the single-threaded oracle on a slice of rows), "
                        "%.1f s" % (threads, dta),
              "single_core": {"value": single["value"], "seconds": single["seconds"], "cores": 1}})
    return d


def cpu_blockscaled_sample(M, N, K, block, budget_rows, seed=0):
    """The oracle on a bounded sample of the block-scaled layer: block-wise
    quantize of `mx` rows of X and `nw` rows of W, then the block-scaled GEMM
    of the sample.  Returns (flops, seconds)."""
    import oracle as O
    import workloads as W
    mx, nw = budget_rows
    rng = np.random.default_rng(seed)
    x = W.f32_to_bf16_bits(rng.standard_normal((mx, K), dtype=np.float32))
    w = W.f32_to_bf16_bits(rng.standard_normal((nw, K), dtype=np.float32) * np.float32(0.02))
    O.lib()
    t = time.perf_counter()
    xq, xs, _ = O.quantize_blockwise(x, O.E4M3, block)
    wq, ws, _ = O.quantize_blockwise(w, O.E4M3, block)
    O.gemm_blockscaled(xq, wq, O.E4M3, xs, ws, block)
    return 2.0 * mx * nw * K, time.perf_counter() - t


def cpu_sweep_sample(rows, cols, seed=0):
    """The oracle quantizing a row sample of the sweep input in every mode;
    returns (algorithmic bytes, seconds)."""
    import oracle as O
    import workloads as W
    x = W.sweep(rows, cols, seed=seed, zero_row=rows // 2)
    O.lib()
    t = time.perf_counter()
    byts = 0
    for fmt in (O.E4M3, O.E5M2):
        for g in (O.PER_TENSOR, O.PER_TOKEN, O.PER_CHANNEL):
            _, s, _ = O.quantize(x, fmt, g)
            byts += rows * cols * 3 + 4 * s.size
    return byts, time.perf_counter() - t


def cpu_blockwise_sample(rows, cols, seed=0):
    """The oracle on a row sample of the block-wise workload; returns
    (algorithmic bytes, seconds)."""
    import oracle as O
    import workloads as W
    x = W.sweep(rows, cols, seed=seed, zero_row=rows // 2)
    O.lib()
    t = time.perf_counter()
    byts = 0
    for fmt, blk, sr in ((O.E4M3, 128, False), (O.E4M3, 32, False), (O.E5M2, 128, True)):
        q, s, _ = O.quantize_blockwise(x, fmt, blk, stochastic=sr, seed=2024)
        byts += rows * cols * 3 + 4 * s.size
        if blk == 128 and fmt == O.E4M3:
            q128, s128 = q, s
    O.dequantize_blockwise(q128, O.E4M3, 128, s128, bf16=True)
    byts += rows * cols * 3 + 4 * s128.size
    return byts, time.perf_counter() - t


def run_reference(args, rank, world):
    if rank != 0:
        return
    cfg = WORKLOADS[args.workload]
    M, N, K = cfg["M"], cfg["N"], cfg["K"]
    if cfg["kind"] in ("sweep", "blockwise"):
        rows = 64
        fn = cpu_sweep_sample if cfg["kind"] == "sweep" else cpu_blockwise_sample
        for _ in range(args.warmup):
            fn(rows, K)
        t = time.perf_counter()
        byts = 0
        for i in range(args.steps):
            byts += fn(rows, K, seed=i)[0]
        dt = time.perf_counter() - t
        value, unit = byts / dt / 1e9, "GB/s"
        sample = ("per step: %d rows x %d cols of the sweep input, %s" %
                  (rows, K, "all six modes" if cfg["kind"] == "sweep" else "the four block-wise calls"))
        dtype = "fp8 codes from bf16, f64 oracle"
    elif cfg["kind"] == "blockscaled":
        rows = (8, 512)
        for _ in range(args.warmup):
            cpu_blockscaled_sample(M, N, K, cfg["block"], rows)
        t = time.perf_counter()
        fl = 0.0
        for i in range(args.steps):
            fl += cpu_blockscaled_sample(M, N, K, cfg["block"], rows, seed=i)[0]
        dt = time.perf_counter() - t
        value, unit = fl / dt / 1e12, "TFLOP/s"
        sample = ("per step: X %d rows x W %d rows (K=%d, block %d), block-wise quantize + exact block-scaled GEMM"
                  % (rows[0], rows[1], K, cfg["block"]))
        dtype = "fp8_e4m3 codes, per-block f32 scales, exact block sums, f64"
    else:
        rows = (8, 512)
        for _ in range(args.warmup):
            cpu_baseline(M, N, K, rows)
        t = time.perf_counter()
        for i in range(args.steps):
            cpu_baseline(M, N, K, rows, seed=i)
        dt = time.perf_counter() - t
        value, unit = 2.0 * rows[0] * rows[1] * K * args.steps / dt / 1e12, "TFLOP/s"
        sample = "per step: X %d rows x W %d rows (K=%d), per-token quantize + exact GEMM" % (rows[0], rows[1], K)
        dtype = "fp8_e4m3 codes, exact integer GEMM, f64"
    line = {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt * 1e3 / max(args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": dtype,
        "data": "synthetic", "config": {"workload": workload_desc(args.workload, cfg), "M": M, "N": N, "K": K,
                                        "parallelism": "rank 0 only"},
        "cpu_baseline": {"value": value, "unit": unit, "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
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
    ap.add_argument("--no-companions", action="store_true",
                    help="default workload only: skip the sweep / MoE / stack lines and the library ceiling")
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
