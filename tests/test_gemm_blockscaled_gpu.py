"""GPU parity of the block-scaled FP8 GEMM (hip-quant README "Block-scaled
Linear and Adafactor Kernel Helpers": FP8 bytes plus FP32 per-block scales of
both operands; "Block-wise FP8 Scaling": scales [..., ceil(K / block_size)])
against the oracle, through the C ABI.

Tolerance (the pass criterion of the scaled GEMM): |out - ref| <=
8e-3 |ref| + 1e-3 max|ref| with ref the exact block sums, scaled and summed
in fp64, rounded once to bf16.  Shapes cover several M and N tiles with
ragged edges, blocks of 32 (four per 128-wide stage) to 256 (two stages per
block), a ragged last K block, K below one block, and K = 0.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from fp8_dynamic_quantization_amax_b200 import _hq as H
from _gpu import assert_gemm_close, dev, dev_bf16, host, host_bits

pytestmark = pytest.mark.gpu

# (M, N, K, block)
SHAPES = [(1, 8, 16, 32), (7, 24, 80, 32), (130, 136, 256, 32), (200, 264, 384, 64), (128, 128, 512, 128),
          (257, 392, 1040, 256), (64, 128, 4096, 32), (300, 520, 272, 96), (129, 256, 2048, 128),
          # more 128 x 128 tiles than SMs: CTAs walk several tiles, so the
          # accumulator and scale rings wrap across tile boundaries (nb = 8:
          # 16-byte scale loads; nb = 7: a partial last chunk of scales)
          (1280, 2048, 256, 32), (1300, 2056, 208, 32)]


def rand_codes(rng, shape, fmt):
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    v = O.decode_array(c.reshape(-1), fmt)
    c.reshape(-1)[~np.isfinite(v)] = 0
    return c


def rand_scales(rng, shape):
    # per-block dequant scales spanning several binades, as amax / fmax gives
    return np.exp(rng.uniform(-8, 2, shape)).astype(np.float32)


@pytest.mark.parametrize("fmt", [O.E4M3, O.E5M2])
@pytest.mark.parametrize("with_bias", [False, True])
def test_blockscaled_gemm_random(fmt, with_bias):
    for i, (M, N, K, block) in enumerate(SHAPES):
        rng = np.random.default_rng(300 + 7 * i + fmt)
        nb = -(-K // block)
        xq, wq = rand_codes(rng, (M, K), fmt), rand_codes(rng, (N, K), fmt)
        xs, ws = rand_scales(rng, (M, nb)), rand_scales(rng, (N, nb))
        bias = W.f32_to_bf16_bits(rng.standard_normal(N).astype(np.float32)) if with_bias else None
        out = H.hq_gemm_blockscaled(dev(xq), dev(wq), dev(xs), dev(ws), fmt, block,
                                    bias=None if bias is None else dev_bf16(bias))
        torch.cuda.synchronize()
        ref = O.gemm_blockscaled(xq, wq, fmt, xs, ws, block, bias)
        assert_gemm_close(host_bits(out), ref)
    H.hq_check_device_error()


def test_blockscaled_gemm_k_zero_writes_the_bias():
    M, N = 5, 16
    bias = W.f32_to_bf16_bits(np.linspace(-3, 3, N).astype(np.float32))
    e = torch.empty((M, 0), dtype=torch.uint8, device="cuda")
    f = torch.empty((N, 0), dtype=torch.uint8, device="cuda")
    s = torch.empty((M, 0), dtype=torch.float32, device="cuda")
    t = torch.empty((N, 0), dtype=torch.float32, device="cuda")
    out = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    H.hq_gemm_blockscaled(e, f, s, t, O.E4M3, 32, bias=dev_bf16(bias), out=out)
    torch.cuda.synchronize()
    assert (host_bits(out) == bias[None, :]).all()
    H.hq_gemm_blockscaled(e, f, s, t, O.E4M3, 32, out=out)
    torch.cuda.synchronize()
    assert (host_bits(out) == 0).all()


def test_blockscaled_gemm_after_blockwise_quantize():
    # the pages' pre-quantized path end to end: bf16 X and W quantized
    # block-wise on the GPU (bit-exact with the oracle), then the GEMM on
    # those codes and scales
    rng = np.random.default_rng(5)
    M, N, K, block = 384, 512, 1024, 32
    xb = W.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    wb = W.f32_to_bf16_bits((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    xq, xs = H.hq_quantize_fp8_blockwise(dev_bf16(xb), O.E4M3, block)
    wq, ws = H.hq_quantize_fp8_blockwise(dev_bf16(wb), O.E4M3, block)
    out = H.hq_gemm_blockscaled(xq, wq, xs, ws, O.E4M3, block)
    torch.cuda.synchronize()
    qx, sx, _ = O.quantize_blockwise(xb, O.E4M3, block)
    qw, sw, _ = O.quantize_blockwise(wb, O.E4M3, block)
    assert np.array_equal(host(xq), qx) and np.array_equal(host(wq), qw)
    assert_gemm_close(host_bits(out), O.gemm_blockscaled(qx, qw, O.E4M3, sx, sw, block))
    # and the block-scaled product tracks the bf16 product within the FP8 error
    exact = W.bf16_bits_to_f32(xb).astype(np.float64) @ W.bf16_bits_to_f32(wb).astype(np.float64).T
    got = W.bf16_bits_to_f32(host_bits(out)).astype(np.float64)
    assert np.abs(got - exact).max() <= 0.05 * np.abs(exact).max()


@pytest.mark.parametrize("block", [32, 128])
def test_blockscaled_gemm_large_sampled(block):
    # a bench-sized product (16 x 64 tiles, K = 8192), checked at sampled
    # entries the oracle computes one by one
    rng = np.random.default_rng(11 + block)
    M, N, K = 2048, 8192, 8192
    nb = K // block
    xq, wq = rand_codes(rng, (M, K), O.E4M3), rand_codes(rng, (N, K), O.E4M3)
    xs, ws = rand_scales(rng, (M, nb)), rand_scales(rng, (N, nb))
    out = host_bits(H.hq_gemm_blockscaled(dev(xq), dev(wq), dev(xs), dev(ws), O.E4M3, block))
    torch.cuda.synchronize()
    ms = np.concatenate([rng.integers(0, M, 200), [0, M - 1, 127, 128]])
    ns = np.concatenate([rng.integers(0, N, 200), [N - 1, 0, 128, 127]])
    ref = O.gemm_blockscaled_entries(xq, wq, O.E4M3, xs, ws, block, ms, ns)
    full_max = np.abs(W.bf16_bits_to_f32(out).astype(np.float64)).max()
    assert_gemm_close(out[ms, ns], ref, max_ref=full_max)
    H.hq_check_device_error()


def test_blockscaled_gemm_overwrites_a_view():
    # caller-owned out: a dense view into a larger buffer is written, the rest untouched
    rng = np.random.default_rng(9)
    M, N, K, block = 40, 64, 256, 64
    xq, wq = rand_codes(rng, (M, K), O.E4M3), rand_codes(rng, (N, K), O.E4M3)
    xs, ws = rand_scales(rng, (M, 4)), rand_scales(rng, (N, 4))
    big = torch.full((M + 8, N), 3.0, dtype=torch.bfloat16, device="cuda")
    view = big[4:4 + M]
    H.hq_gemm_blockscaled(dev(xq), dev(wq), dev(xs), dev(ws), O.E4M3, block, out=view)
    torch.cuda.synchronize()
    assert_gemm_close(host_bits(view), O.gemm_blockscaled(xq, wq, O.E4M3, xs, ws, block))
    b = host_bits(big)
    assert (b[:4] == b[0, 0]).all() and (b[4 + M:] == b[0, 0]).all()


def test_blockscaled_gemm_empty_is_a_no_op():
    # M == 0: OK with no launch, null A and x_scales allowed
    w = torch.zeros((16, 64), dtype=torch.uint8, device="cuda")
    s = torch.ones((16, 2), dtype=torch.float32, device="cuda")
    out = torch.zeros((1, 16), dtype=torch.bfloat16, device="cuda")
    assert H.lib.hq_gemm_blockscaled(None, w.data_ptr(), O.E4M3, None, s.data_ptr(), 32, None, 0, 16, 64,
                                     out.data_ptr(), None) == 0
    torch.cuda.synchronize()
    assert (host_bits(out) == 0).all()


def test_linear_blockwise_is_quantize_then_gemm():
    # the convenience path equals the three calls it chains, bit for bit, and
    # tracks the bf16 product within the FP8 error
    rng = np.random.default_rng(21)
    M, N, K, block = 96, 264, 512, 32
    xb = W.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    wb = W.f32_to_bf16_bits((rng.standard_normal((N, K)) * 0.05).astype(np.float32))
    bias = W.f32_to_bf16_bits(rng.standard_normal(N).astype(np.float32))
    x, w, b = dev_bf16(xb), dev_bf16(wb), dev_bf16(bias)
    out = H.hq_linear_blockwise(x, w, bias=b, block=block)
    xq, xs = H.hq_quantize_fp8_blockwise(x, O.E4M3, block)
    wq, ws = H.hq_quantize_fp8_blockwise(w, O.E4M3, block)
    ref = H.hq_gemm_blockscaled(xq, wq, xs, ws, O.E4M3, block, bias=b)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    qx, sx, _ = O.quantize_blockwise(xb, O.E4M3, block)
    qw, sw, _ = O.quantize_blockwise(wb, O.E4M3, block)
    assert_gemm_close(host_bits(out), O.gemm_blockscaled(qx, qw, O.E4M3, sx, sw, block, bias))
