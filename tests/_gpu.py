"""Shared helpers for the GPU parity tests (moving seeded host arrays to the
device and back, and the GEMM tolerance).  Holds none of the method's
arithmetic."""
import numpy as np
import torch

import workloads as W

# GEMM pass criterion: |out - ref| <= 8e-3 |ref| + 1e-3 max|ref|, where ref is
# the exact dequantized product rounded once to bf16 (the oracle's output).
REL_TOL = 8e-3
ABS_TOL_FRAC = 1e-3


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 bit patterns on the host."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy()


def assert_gemm_close(out_bits: np.ndarray, ref_bits: np.ndarray, max_ref=None):
    out = W.bf16_bits_to_f32(out_bits).astype(np.float64)
    ref = W.bf16_bits_to_f32(ref_bits).astype(np.float64)
    assert out.shape == ref.shape
    assert np.isfinite(ref).all()
    if max_ref is None:
        max_ref = np.abs(ref).max() if ref.size else 0.0
    tol = REL_TOL * np.abs(ref) + ABS_TOL_FRAC * max_ref
    err = np.abs(out - ref)
    bad = ~(err <= tol)
    if bad.any():
        i = np.argmax(np.where(bad, err - tol, -np.inf))
        raise AssertionError("%d of %d outputs outside tolerance; worst at flat %d: out %r ref %r tol %r"
                             % (bad.sum(), bad.size, i, out.reshape(-1)[i], ref.reshape(-1)[i], tol.reshape(-1)[i]))
