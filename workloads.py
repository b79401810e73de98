"""Seeded synthetic inputs for the five workloads (shared by the tests, the
benchmark and the oracle legs).

This module draws random numbers and lays them out; it holds none of the
quantization or GEMM arithmetic.  bf16 tensors are returned as uint16 bit
patterns, rounded from float32 samples to nearest-even by torch's CPU cast.

Workload recipes (the benchmark configurations' sizes and distributions;
details they leave open are this module's readings):
  tiny      X f32 [64,256] ~N(0,1), rows 3 and 17 scaled x50;
            W f32 [128,256] ~N(0,0.02); seed 0.
  sweep     bf16 [8192,8192] ~N(0,1); 0.1% of positions x100; a further 0.1%
            set to +0.0 (the first 64 of them -0.0); row 4321 all zero.
  delayed   X_t bf16 [2048,1024] = std_t * N(0,1), std_t = 0.5*16^(t/199),
            seed (0, t); W_up [4096,1024] (seed 1), W_down [1024,4096]
            (seed 2) ~N(0,0.02).
  large     X bf16 [M,8192] ~N(0,1) (seed 0); W bf16 [N,K] ~N(0,0.02) (seed 1).
  moe       64 experts, K=2048, N=1408, 32768 tokens; Zipf(1.1) counts over
            62 ranks, largest-remainder rounding, 2 experts empty.
"""
import numpy as np
import torch


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def normal(shape, std, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


# ----------------------------------------------------------------- tiny
def tiny(M=64, N=128, K=256, seed=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K), dtype=np.float32)
    for r in (3, 17):
        if r < M:
            x[r] *= np.float32(50.0)
    w = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    return x, w


# ---------------------------------------------------------------- sweep
def sweep(rows=8192, cols=8192, seed=0, outlier_frac=0.001, zero_frac=0.001,
          neg_zeros=64, zero_row=4321):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols), dtype=np.float32)
    flat = x.reshape(-1)
    n = flat.size
    n_out = int(round(n * outlier_frac))
    idx = rng.choice(n, size=n_out, replace=False)
    flat[idx] *= np.float32(100.0)
    n_zero = int(round(n * zero_frac))
    zidx = rng.choice(n, size=n_zero, replace=False)
    flat[zidx] = np.float32(0.0)
    flat[zidx[:min(neg_zeros, n_zero)]] = np.float32(-0.0)
    x[zero_row % rows, :] = 0.0
    return f32_to_bf16_bits(x)


# -------------------------------------------------------------- delayed
def delayed_std(t, steps=200):
    return 0.5 * 16.0 ** (t / (steps - 1))


def delayed_x(t, tokens=2048, dim=1024, steps=200):
    rng = np.random.default_rng([0, t])
    x = rng.standard_normal((tokens, dim), dtype=np.float32)
    x *= np.float32(delayed_std(t, steps))
    return f32_to_bf16_bits(x)


def delayed_weights(dim=1024, hidden=4096):
    w_up = f32_to_bf16_bits(normal((hidden, dim), 0.02, 1))
    w_down = f32_to_bf16_bits(normal((dim, hidden), 0.02, 2))
    return w_up, w_down


# ---------------------------------------------------------------- large
def large_x(M, K=8192, seed=0):
    return f32_to_bf16_bits(normal((M, K), 1.0, seed))


def large_w(N=28672, K=8192, seed=1):
    return f32_to_bf16_bits(normal((N, K), 0.02, seed))


# ------------------------------------------------------------------ moe
def zipf_counts(total=32768, ranks=62, s=1.1):
    r = np.arange(1, ranks + 1, dtype=np.float64)
    w = r ** (-s)
    ideal = total * w / w.sum()
    base = np.floor(ideal).astype(np.int64)
    rem = total - int(base.sum())
    order = np.argsort(-(ideal - base), kind="stable")
    base[order[:rem]] += 1
    return base


def moe_offsets(experts=64, total=32768, empty=(7, 41), s=1.1, seed=0):
    """Exclusive prefix sum [experts+1] of per-expert row counts."""
    live = [e for e in range(experts) if e not in empty]
    counts_by_rank = zipf_counts(total, len(live), s)
    rng = np.random.default_rng(seed)
    perm = rng.permutation(len(live))
    counts = np.zeros(experts, np.int64)
    for rank, slot in enumerate(perm):
        counts[live[slot]] = counts_by_rank[rank]
    off = np.zeros(experts + 1, np.int32)
    off[1:] = np.cumsum(counts)
    return off


def moe_inputs(experts=64, tokens=32768, N=1408, K=2048, seed=0, empty=(7, 41)):
    off = moe_offsets(experts, tokens, empty, seed=seed)
    x = f32_to_bf16_bits(normal((tokens, K), 1.0, seed))
    w = f32_to_bf16_bits(normal((experts, N, K), 0.02, seed + 1))
    return x, w, off


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)
