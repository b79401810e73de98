"""GPU parity of the GEMM's fused epilogues (hq_gemm_a8w8_ex), through the C
ABI: the bias added before the bf16 rounding (AstrAI ops.cu
linear_forward_fp8) and the FP8 output (mm_fp8's out_dtype 1), here the
delayed per-tensor quantize of the bf16 result with an amax-history ring.

The FP8 output must be bit-identical to the two calls it fuses, hq_gemm_a8w8
(with the bias) followed by hq_quantize_fp8 with the same ring: codes, dequant
scale, amax and the ring after every step.  Against the oracle (its GEMM, then
its delayed quantize, fed only generator inputs), the codes must agree
wherever the GPU's bf16 result equals the oracle's; the bias path is checked
within the GEMM tolerance.
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

# (M, N, K): 1-CTA 128-wide tiles, the CTA pair (256 x 256), the 256 x 512
# pair tile (M >= 8192, N % 512 == 0), the 1-CTA 256-wide tile and a decode
# tile, each with a ragged edge somewhere
SHAPES = [(300, 272, 144), (700, 2048, 128), (8200, 2048, 32), (260, 2304, 96), (16, 2080, 256)]


def rand_codes(rng, shape, fmt):
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    v = O.decode_array(c.reshape(-1), fmt)
    c.reshape(-1)[~np.isfinite(v)] = 0
    return c


def operands(i, M, N, K, fmt):
    rng = np.random.default_rng(500 + i)
    xq, wq = rand_codes(rng, (M, K), fmt), rand_codes(rng, (N, K), fmt)
    xs = rng.uniform(0.001, 0.01, M).astype(np.float32)
    ws = rng.uniform(0.001, 0.01, N).astype(np.float32)
    if fmt == O.E5M2:
        xs *= np.float32(1e-4)
        ws *= np.float32(1e-4)
    bias = W.f32_to_bf16_bits(rng.standard_normal(N).astype(np.float32) * np.float32(0.5))
    return xq, wq, xs, ws, bias


def fresh_ring(scale=1.0):
    r = np.zeros(L + 2, np.float32)
    r[L] = scale
    return r


@pytest.mark.parametrize("fmt", [O.E4M3, O.E5M2])
def test_bias_bf16_out(fmt):
    for i, (M, N, K) in enumerate(SHAPES):
        xq, wq, xs, ws, bias = operands(i, M, N, K, fmt)
        out = H.hq_gemm_a8w8_ex(dev(xq), dev(wq), dev(xs), dev(ws), fmt, bias=dev(bias))
        torch.cuda.synchronize()
        assert_gemm_close(host_bits(out), O.gemm_a8w8_bias(xq, wq, fmt, xs, ws, bias))
    H.hq_check_device_error()


@pytest.mark.parametrize("with_bias", [False, True])
@pytest.mark.parametrize("q_fmt", [H.E4M3, H.E5M2])
def test_fp8_out_equals_gemm_then_delayed_quantize(q_fmt, with_bias):
    for i, (M, N, K) in enumerate(SHAPES):
        xq, wq, xs, ws, bias = operands(i, M, N, K, O.E4M3)
        xq_d, wq_d, xs_d, ws_d = dev(xq), dev(wq), dev(xs), dev(ws)
        b_d = dev(bias) if with_bias else None
        ring_f = torch.from_numpy(fresh_ring()).cuda()
        ring_u = ring_f.clone()
        ws_f = torch.zeros(256, dtype=torch.uint8, device="cuda")
        for step in range(3):  # the ring's multiplier changes after the first step
            if step:
                xq_d = dev(rand_codes(np.random.default_rng(900 + 10 * i + step), (M, K), O.E4M3))
            a_f = torch.full((1,), -1.0, device="cuda")
            q_f, s_f = H.hq_gemm_a8w8_ex(xq_d, wq_d, xs_d, ws_d, H.E4M3, bias=b_d, q_fmt=q_fmt, q_amax=a_f,
                                         ring=ring_f, ring_idx=step, workspace=ws_f)
            h = H.hq_gemm_a8w8_ex(xq_d, wq_d, xs_d, ws_d, H.E4M3, bias=b_d)
            a_u = torch.full((1,), -1.0, device="cuda")
            q_u, s_u = H.hq_quantize_fp8(h, q_fmt, H.PER_TENSOR, amax_out=a_u, ring=ring_u, ring_idx=step)
            torch.cuda.synchronize()
            assert torch.equal(q_f, q_u), "codes %s step %d" % ((M, N, K), step)
            assert torch.equal(s_f.view(torch.int32), s_u.view(torch.int32))
            assert torch.equal(a_f.view(torch.int32), a_u.view(torch.int32))
            assert torch.equal(ring_f.view(torch.int32), ring_u.view(torch.int32))
            assert (host(ws_f) == 0).all()
    H.hq_check_device_error()


@pytest.mark.parametrize("q_fmt", [O.E4M3, O.E5M2])
def test_fp8_out_vs_oracle(q_fmt):
    for i, (M, N, K) in enumerate(SHAPES[:4]):
        xq, wq, xs, ws, bias = operands(i, M, N, K, O.E4M3)
        ring = fresh_ring(0.75)  # a multiplier that is not 1
        ring_d = torch.from_numpy(ring.copy()).cuda()
        a_d = torch.zeros(1, device="cuda")
        q_d, s_d = H.hq_gemm_a8w8_ex(dev(xq), dev(wq), dev(xs), dev(ws), H.E4M3, bias=dev(bias), q_fmt=q_fmt,
                                     q_amax=a_d, ring=ring_d, ring_idx=3)
        h_gpu = H.hq_gemm_a8w8_ex(dev(xq), dev(wq), dev(xs), dev(ws), H.E4M3, bias=dev(bias))
        torch.cuda.synchronize()
        # oracle, fed only generator inputs: its GEMM (bias), then its delayed quantize
        h_ref = O.gemm_a8w8_bias(xq, wq, O.E4M3, xs, ws, bias)
        q_ref, s_ref, a_ref = O.quantize(h_ref, q_fmt, O.PER_TENSOR, ring=ring, ring_idx=3)
        hb = host_bits(h_gpu)
        assert_gemm_close(hb, h_ref)
        same = hb == h_ref
        assert same.mean() > 0.99
        np.testing.assert_array_equal(host(q_d)[same], q_ref[same])
        np.testing.assert_array_equal(host(s_d).view(np.uint32), s_ref.view(np.uint32))  # 1/m of the entry ring
        a = float(host(a_d)[0])
        assert abs(a - float(a_ref[0])) <= 8e-3 * abs(float(a_ref[0]))
        if a == float(a_ref[0]):
            np.testing.assert_array_equal(host(ring_d).view(np.uint32), ring.view(np.uint32))
    H.hq_check_device_error()


def test_fp8_out_empty_steps_the_ring():
    # M == 0: the delayed quantize of an empty result (amax 0) still steps the ring
    ring_f = torch.from_numpy(fresh_ring(2.0)).cuda()
    ring_f[:L] = torch.arange(1, L + 1, dtype=torch.float32)
    ring_u = ring_f.clone()
    xq = torch.zeros((0, 64), dtype=torch.uint8, device="cuda")
    wq = torch.zeros((32, 64), dtype=torch.uint8, device="cuda")
    q_f, s_f = H.hq_gemm_a8w8_ex(xq, wq, torch.ones(1, device="cuda"), torch.ones(1, device="cuda"), H.E4M3,
                                 ring=ring_f, ring_idx=L - 1)
    q_u, s_u = H.hq_quantize_fp8(torch.zeros((0, 32), dtype=torch.bfloat16, device="cuda"), H.E4M3, H.PER_TENSOR,
                                 ring=ring_u, ring_idx=L - 1)
    torch.cuda.synchronize()
    assert torch.equal(ring_f, ring_u) and torch.equal(s_f, s_u)
    assert float(host(ring_f)[L - 1]) == 0.0


@pytest.mark.parametrize("q_fmt", [O.E4M3, O.E5M2])
def test_fp8_out_ring_keeps_scale_when_next_not_finite(q_fmt):
    # The ring publishes next = f32(fmax / win) * 2^-margin only when next is
    # finite and > 0 (the delayed-scaling step of AstrAI ops.cu, with the
    # guard of hip-quant's "Training-path numerical guards").  Three ring
    # states reach the guard, one control publishes:
    #   a subnormal window (hist holds 2^-140, the result is all zero):
    #     fmax / 2^-140 overflows to +Inf
    #   margin -126 on a result of amax 44: next overflows to +Inf
    #   margin 126 with 2^127 in the window: next underflows to 0
    M, N, K = 300, 272, 144
    xq, wq, xs, ws, _ = operands(7, M, N, K, O.E4M3)
    zeros = np.zeros_like(xq)
    cases = [("subnormal window", zeros, 2.0 ** -140, 0, False),
             ("margin -126", xq, 0.0, -126, False),
             ("margin 126", xq, 2.0 ** 127, 126, False),
             ("control", xq, 0.0, 0, True)]
    for name, x_codes, preset, margin, publishes in cases:
        ring = fresh_ring(0.75)
        ring[5] = np.float32(preset)
        ring_f = torch.from_numpy(ring.copy()).cuda()
        ring_u = ring_f.clone()
        args = (dev(x_codes), dev(wq), dev(xs), dev(ws), H.E4M3)
        q_f, s_f = H.hq_gemm_a8w8_ex(*args, q_fmt=q_fmt, ring=ring_f, ring_idx=2, ring_margin=margin)
        h = H.hq_gemm_a8w8_ex(*args)
        q_u, s_u = H.hq_quantize_fp8(h, q_fmt, H.PER_TENSOR, ring=ring_u, ring_idx=2, ring_margin=margin)
        torch.cuda.synchronize()
        assert torch.equal(q_f, q_u), name
        assert torch.equal(ring_f.view(torch.int32), ring_u.view(torch.int32)), name
        # the oracle's delayed quantize of the GPU's own bf16 result
        ring_o = ring.copy()
        q_o, s_o, _ = O.quantize(host_bits(h), q_fmt, O.PER_TENSOR, ring=ring_o, ring_idx=2, ring_margin=margin)
        np.testing.assert_array_equal(host(q_f), q_o)
        np.testing.assert_array_equal(host(s_f).view(np.uint32), s_o.view(np.uint32))
        np.testing.assert_array_equal(host(ring_f).view(np.uint32), ring_o.view(np.uint32))
        kept = host(ring_f)[L] == np.float32(0.75)
        assert kept != publishes, name
    H.hq_check_device_error()


# ---------------------------------------------------------------- block-wise FP8 output
# hq_gemm_a8w8_blockq: the bf16 result quantized in 32-column blocks of a row
# by the epilogue (hip-quant README "Block-wise FP8 Scaling" on the output of
# mm_fp8).  Shapes with N % 32 == 0: the 1-CTA tiles, the 256 x 256 CTA pair
# (M >= 4096, N % 512 != 0), the 256 x 512 pair tile, a 256-wide 1-CTA tile
# and a decode tile; ragged M everywhere.
BQ_SHAPES = [(300, 288, 144), (700, 2048, 128), (4200, 1280, 64), (8200, 2048, 32), (260, 2304, 96),
             (16, 2080, 256)]


def _blockq_pair(i, M, N, K, q_fmt, with_bias, big_rows=()):
    """The fused call and the two calls it fuses, on the same operands."""
    xq, wq, xs, ws, bias = operands(40 + i, M, N, K, O.E4M3)
    for r in big_rows:  # rows whose bf16 result overflows to +-Inf in places
        xs[r] = np.float32(3e38)
    xq_d, wq_d, xs_d, ws_d = dev(xq), dev(wq), dev(xs), dev(ws)
    b_d = dev(bias) if with_bias else None
    q, s = H.hq_gemm_a8w8_blockq(xq_d, wq_d, xs_d, ws_d, H.E4M3, bias=b_d, q_fmt=q_fmt)
    h = H.hq_gemm_a8w8_ex(xq_d, wq_d, xs_d, ws_d, H.E4M3, bias=b_d)
    q2, s2 = H.hq_quantize_fp8_blockwise(h, q_fmt, 32)
    torch.cuda.synchronize()
    return (xq, wq, xs, ws, bias), q, s, h, q2, s2


@pytest.mark.parametrize("with_bias", [False, True])
@pytest.mark.parametrize("q_fmt", [H.E4M3, H.E5M2])
def test_blockwise_out_equals_gemm_then_blockwise_quantize(q_fmt, with_bias):
    for i, (M, N, K) in enumerate(BQ_SHAPES):
        _, q, s, _, q2, s2 = _blockq_pair(i, M, N, K, q_fmt, with_bias)
        assert s.shape == (M, N // 32)
        assert np.array_equal(host(q), host(q2)), (M, N, K)
        assert np.array_equal(host(s).view(np.uint32), host(s2).view(np.uint32)), (M, N, K)
    H.hq_check_device_error()


@pytest.mark.parametrize("q_fmt", [H.E4M3, H.E5M2])
def test_blockwise_out_vs_oracle(q_fmt):
    # stage-wise: the oracle's GEMM within the GEMM tolerance, then the
    # oracle's block-wise quantize of the GPU's bf16 result bit for bit
    for i, (M, N, K) in enumerate(BQ_SHAPES[:3] + BQ_SHAPES[4:]):
        (xq, wq, xs, ws, bias), q, s, h, _, _ = _blockq_pair(i, M, N, K, q_fmt, True)
        hb = host_bits(h)
        assert_gemm_close(hb, O.gemm_a8w8_bias(xq, wq, O.E4M3, xs, ws, bias))
        qo, so, _ = O.quantize_blockwise(hb, q_fmt, 32)
        assert np.array_equal(host(q), qo), (M, N, K)
        assert np.array_equal(host(s).view(np.uint32), so.view(np.uint32)), (M, N, K)
    H.hq_check_device_error()


def test_blockwise_out_non_finite_results():
    # rows whose scaled result overflows: +-Inf entries leave the block
    # maxima (finite-only amax) and saturate; an all-Inf block keeps m = 1
    for i, (M, N, K) in enumerate([(300, 288, 144), (4200, 1280, 64)]):
        _, q, s, h, q2, s2 = _blockq_pair(i, M, N, K, H.E4M3, False, big_rows=(0, 5, 131))
        hb = host_bits(h)
        assert (np.abs(W.bf16_bits_to_f32(hb[[0, 5, 131]])) == np.inf).any()
        assert np.array_equal(host(q), host(q2))
        assert np.array_equal(host(s).view(np.uint32), host(s2).view(np.uint32))
        qo, so, _ = O.quantize_blockwise(hb, H.E4M3, 32)
        assert np.array_equal(host(q), qo) and np.array_equal(host(s).view(np.uint32), so.view(np.uint32))
    H.hq_check_device_error()


def test_blockwise_out_feeds_the_blockscaled_gemm():
    # h's codes and scales are the next layer's block-scaled A operand (K = N)
    M, N, K, N2 = 700, 2048, 128, 384
    (xq, wq, xs, ws, bias), q, s, h, _, _ = _blockq_pair(2, M, N, K, H.E4M3, True)
    rng = np.random.default_rng(77)
    w2 = W.f32_to_bf16_bits(rng.standard_normal((N2, N)).astype(np.float32) * np.float32(0.02))
    w2q, w2s = H.hq_quantize_fp8_blockwise(dev_bf16(w2), H.E4M3, 32)
    y = H.hq_gemm_blockscaled(q, w2q, s, w2s, H.E4M3, 32)
    torch.cuda.synchronize()
    assert_gemm_close(host_bits(y), O.gemm_blockscaled(host(q), host(w2q), H.E4M3, host(s), host(w2s), 32))
    H.hq_check_device_error()


def test_blockwise_out_empty():
    xq = torch.zeros((0, 64), dtype=torch.uint8, device="cuda")
    wq = torch.zeros((64, 64), dtype=torch.uint8, device="cuda")
    xs = torch.ones(1, device="cuda")
    q, s = H.hq_gemm_a8w8_blockq(xq, wq, xs, torch.ones(64, device="cuda"), H.E4M3)
    assert q.shape == (0, 64) and s.shape == (0, 2)
