"""GPU parity of the backward path's quantize (AstrAI ops.cu
linear_backward_fp8): per-tensor FP8 codes written row-major and
transposed, in the dynamic, delayed-ring and static-multiplier forms, then
dX = g @ w and dW = g^T @ x as NT GEMMs on the transposed codes.

The oracle quantizes with its own functions (the static form through a
scratch ring whose scale slot holds the multiplier) and transposes with
numpy; codes, scales, amax and rings must be bit-exact.  The two GEMMs are
compared with the oracle's GEMM of the oracle's codes, within the GEMM
tolerance.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from fp8_dynamic_quantization_amax_b200 import _hq as H
from _gpu import assert_gemm_close, dev, dev_bf16, host, host_bits

pytestmark = pytest.mark.gpu
L = 16
SHAPES = [(16, 16), (48, 80), (64, 64), (144, 208), (1040, 528)]


def make(shape, dtype, seed, specials=True):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal(shape) * rng.uniform(0.1, 20)).astype(np.float32)
    if specials and x.size >= 16:
        idx = rng.choice(x.size, 6, replace=False)
        x.reshape(-1)[idx] = np.array([np.nan, np.inf, -np.inf, -0.0, 1e-40, 6e4], np.float32)
    if dtype == "f32":
        return x, torch.from_numpy(x).cuda()
    if dtype == "bf16":
        b = W.f32_to_bf16_bits(x)
        return b, dev_bf16(b)
    h = x.astype(np.float16)
    return h, torch.from_numpy(h).cuda()


def oracle_codes(xh, fmt, mode, ring=None, idx=0, mult=None):
    if mode == "dynamic":
        return O.quantize(xh, fmt, O.PER_TENSOR)
    if mode == "delayed":
        return O.quantize(xh, fmt, O.PER_TENSOR, ring=ring, ring_idx=idx)
    scratch = np.zeros(L + 2, np.float32)  # static: the multiplier in a ring that is then dropped
    scratch[L] = mult
    return O.quantize(xh, fmt, O.PER_TENSOR, ring=scratch, ring_idx=0)


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("mode", ["dynamic", "delayed", "static"])
@pytest.mark.parametrize("fmt", [O.E4M3, O.E5M2])
def test_quantize_transpose_bit_exact(dtype, mode, fmt):
    for i, shape in enumerate(SHAPES):
        xh, xd = make(shape, dtype, seed=700 + 10 * i + fmt)
        ring = np.zeros(L + 2, np.float32)
        ring[:L] = np.linspace(0.5, 9.0, L).astype(np.float32)
        ring[L] = 3.0
        ring_d = torch.from_numpy(ring.copy()).cuda() if mode == "delayed" else None
        mult = np.float32(0.37 if fmt == O.E4M3 else 11.0)
        mult_d = torch.tensor([mult], dtype=torch.float32, device="cuda") if mode == "static" else None
        ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
        amax = torch.full((1,), -1.0, device="cuda")
        q, qt, s = H.hq_quantize_fp8_transpose(xd, fmt, q=True, multiplier=mult_d, amax_out=amax, ring=ring_d,
                                               ring_idx=5, workspace=ws)
        torch.cuda.synchronize()
        qo, so, ao = oracle_codes(xh, fmt, mode, ring=ring, idx=5, mult=mult)
        np.testing.assert_array_equal(host(q), qo, err_msg="q %s %s %s" % (shape, dtype, mode))
        np.testing.assert_array_equal(host(qt), qo.T, err_msg="qt %s %s %s" % (shape, dtype, mode))
        np.testing.assert_array_equal(host(s).view(np.uint32), so.view(np.uint32))
        np.testing.assert_array_equal(host(amax).view(np.uint32), ao.view(np.uint32))
        if mode == "delayed":
            np.testing.assert_array_equal(host(ring_d).view(np.uint32), ring.view(np.uint32))
        assert (host(ws) == 0).all()
    H.hq_check_device_error()


def test_quantize_transpose_full_size():
    # the quantize sweep's input, dynamic E5M2 (the gradient format)
    xb = W.sweep()
    q0, qt, s = H.hq_quantize_fp8_transpose(dev_bf16(xb), O.E5M2, q=True)
    torch.cuda.synchronize()
    qo, so, _ = O.quantize(xb, O.E5M2, O.PER_TENSOR)
    assert np.array_equal(host(q0), qo)
    assert np.array_equal(host(qt), qo.T)
    assert host(s).view(np.uint32)[0] == so.view(np.uint32)[0]
    H.hq_check_device_error()


@pytest.mark.parametrize("fmt", [O.E4M3, O.E5M2])
def test_backward_gemms_vs_oracle(fmt):
    # g [M, N] with a delayed ring, w [N, K] and x [M, K] with the forward's
    # multipliers (static); dX = g @ w, dW = g^T @ x on the transposed codes
    M, N, K = 272, 384, 528
    rng = np.random.default_rng(41 + fmt)
    g = W.f32_to_bf16_bits(rng.standard_normal((M, N)).astype(np.float32) * np.float32(1e-3))
    x = W.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    w = W.f32_to_bf16_bits(rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02))
    ring = np.zeros(L + 2, np.float32)
    ring[L] = np.float32(O.fmax(fmt) / 4e-3)
    ring_d = torch.from_numpy(ring.copy()).cuda()
    mw = np.float32(O.multiplier(float(np.abs(W.bf16_bits_to_f32(w)).max()), fmt))
    mx = np.float32(O.multiplier(float(np.abs(W.bf16_bits_to_f32(x)).max()), fmt))
    g8, gT8, sg = H.hq_quantize_fp8_transpose(dev_bf16(g), fmt, q=True, ring=ring_d, ring_idx=0)
    _, wT8, sw = H.hq_quantize_fp8_transpose(dev_bf16(w), fmt, multiplier=torch.tensor([mw], device="cuda"))
    _, xT8, sx = H.hq_quantize_fp8_transpose(dev_bf16(x), fmt, multiplier=torch.tensor([mx], device="cuda"))
    dX = H.hq_gemm_a8w8(g8, wT8, sg, sw, fmt)     # [M, K] = g [M, N] . (w^T)[K, N]^T
    dW = H.hq_gemm_a8w8(gT8, xT8, sg, sx, fmt)    # [N, K] = (g^T)[N, M] . (x^T)[K, M]^T
    torch.cuda.synchronize()
    go, gso, _ = oracle_codes(g, fmt, "delayed", ring=ring, idx=0)
    wo, wso, _ = oracle_codes(w, fmt, "static", mult=mw)
    xo, xso, _ = oracle_codes(x, fmt, "static", mult=mx)
    assert np.array_equal(host(gT8), go.T) and np.array_equal(host(wT8), wo.T) and np.array_equal(host(xT8), xo.T)
    assert_gemm_close(host_bits(dX), O.gemm_a8w8(go, np.ascontiguousarray(wo.T), fmt, gso, wso))
    assert_gemm_close(host_bits(dW), O.gemm_a8w8(np.ascontiguousarray(go.T), np.ascontiguousarray(xo.T), fmt,
                                                 gso, xso))
    np.testing.assert_array_equal(host(ring_d).view(np.uint32), ring.view(np.uint32))
    H.hq_check_device_error()
