"""GPU parity of the block-wise FP8 quantize and dequantize (hip-quant README
"Block-wise FP8 Scaling") against the oracle, through the C ABI: codes, block
dequant scales and block amax bit-exact for both formats, every input type,
round-to-nearest-even and stochastic rounding, blocks that divide the row and
ragged last blocks; dequantized values bit-exact in f32 and bf16.

Inputs mix a wide dynamic range (so that neighbouring blocks get very
different scales, and some blocks are all zero), plus NaN, +-Inf, -0 and f32
subnormals.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from fp8_dynamic_quantization_amax_b200 import _hq as H
from _gpu import dev, dev_bf16, host, host_bits

pytestmark = pytest.mark.gpu
# (rows, cols, block): blocks dividing the row, ragged last blocks, a block
# wider than the row (the per-token case), a single row of 16; power-of-two
# blocks of 16 .. 2048 (one to eight warp-wide vectors per block), blocks of
# 48 and 80 elements, and rows too long for a shared-memory stage pair.
CASES = [(1, 16, 16), (7, 48, 32), (33, 272, 128), (130, 1024, 128), (5, 8208, 64), (9, 96, 256), (64, 4096, 32),
         (6, 192, 48), (3, 480, 80), (4, 2064, 512), (3, 3008, 1024), (2, 4608, 2048), (3, 40000, 128)]


def make(shape, dtype, seed, specials=True):
    rng = np.random.default_rng(seed)
    rows, cols = shape
    # per-16-column magnitude bands so that blocks differ in scale
    band = np.exp(rng.uniform(-14, 6, (rows, (cols + 15) // 16))).repeat(16, axis=1)[:, :cols]
    x = (rng.standard_normal(shape) * band).astype(np.float32)
    if cols >= 32 and rows >= 2:
        x[1, :16] = 0.0                                   # an all-zero block part
    flat = x.reshape(-1)
    if specials and flat.size >= 16:
        idx = rng.choice(flat.size, 8, replace=False)
        flat[idx] = np.array([np.nan, np.inf, -np.inf, -0.0, 0.0, 1e-40, -3e-41, 5e4], np.float32)
    if dtype == "f32":
        return x, torch.from_numpy(x).cuda()
    if dtype == "bf16":
        b = W.f32_to_bf16_bits(x)
        return b, dev_bf16(b)
    h = x.astype(np.float16)
    return h, torch.from_numpy(h).cuda()


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("fmt", [O.E4M3, O.E5M2])
def test_blockwise_quantize_bit_exact(dtype, fmt):
    for i, (rows, cols, block) in enumerate(CASES):
        xh, xd = make((rows, cols), dtype, seed=900 + 10 * i + fmt)
        a = torch.full((rows, -(-cols // block)), -1.0, device="cuda")
        q, s = H.hq_quantize_fp8_blockwise(xd, fmt, block, amax_out=a)
        torch.cuda.synchronize()
        qo, so, ao = O.quantize_blockwise(xh, fmt, block)
        msg = "%s %s fmt %d" % ((rows, cols, block), dtype, fmt)
        np.testing.assert_array_equal(host(q), qo, err_msg="codes " + msg)
        np.testing.assert_array_equal(host(s).view(np.uint32), so.view(np.uint32), err_msg="scales " + msg)
        np.testing.assert_array_equal(host(a).view(np.uint32), ao.view(np.uint32), err_msg="amax " + msg)
    H.hq_check_device_error()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_blockwise_stochastic_e5m2_bit_exact(dtype):
    for i, (rows, cols, block) in enumerate(CASES):
        xh, xd = make((rows, cols), dtype, seed=950 + i)
        seed = (0xD1B54A32D192ED03 * (i + 3)) & ((1 << 64) - 1)
        q, s = H.hq_quantize_fp8_blockwise(xd, O.E5M2, block, stochastic=True, seed=seed)
        torch.cuda.synchronize()
        qo, so, _ = O.quantize_blockwise(xh, O.E5M2, block, stochastic=True, seed=seed)
        np.testing.assert_array_equal(host(q), qo, err_msg="codes %s" % ((rows, cols, block),))
        np.testing.assert_array_equal(host(s).view(np.uint32), so.view(np.uint32))
    H.hq_check_device_error()


def test_blockwise_wide_block_is_per_token():
    # One block per row: the same codes and scales as the per-token quantize.
    xh, xd = make((40, 320), "bf16", seed=5, specials=False)
    q, s = H.hq_quantize_fp8_blockwise(xd, O.E4M3, 512)
    qt, st = H.hq_quantize_fp8(xd, O.E4M3, O.PER_TOKEN)
    torch.cuda.synchronize()
    assert torch.equal(q, qt)
    assert torch.equal(s.reshape(-1), st.reshape(-1))


def _same_or_both_nan(got, ref, bf16):
    if bf16:
        g = W.bf16_bits_to_f32(got)
        r = W.bf16_bits_to_f32(ref)
    else:
        g, r = got, ref
    nan = np.isnan(r)
    assert (np.isnan(g) == nan).all()
    bits = np.uint16 if bf16 else np.uint32
    np.testing.assert_array_equal(got[~nan].view(bits), ref[~nan].view(bits))


@pytest.mark.parametrize("fmt", [O.E4M3, O.E5M2])
@pytest.mark.parametrize("bf16", [False, True])
def test_blockwise_dequantize_bit_exact(fmt, bf16):
    for i, (rows, cols, block) in enumerate(CASES):
        rng = np.random.default_rng(970 + i)
        qh = rng.integers(0, 256, (rows, cols), dtype=np.uint8)       # every code, NaN and Inf included
        nb = -(-cols // block)
        sh = np.exp(rng.uniform(-20, 20, (rows, nb))).astype(np.float32)
        out = H.hq_dequantize_fp8_blockwise(dev(qh), dev(sh), fmt, block,
                                            out_dtype=torch.bfloat16 if bf16 else torch.float32)
        torch.cuda.synchronize()
        ref = O.dequantize_blockwise(qh, fmt, block, sh, bf16=bf16)
        got = host_bits(out) if bf16 else host(out)
        if bf16:
            _same_or_both_nan(got, ref, True)
        else:
            _same_or_both_nan(got.view(np.float32), ref, False)
    H.hq_check_device_error()


def test_blockwise_round_trip_error_bound():
    # Dequantized E4M3 codes are within half a step (2^-4 relative for normal
    # codes, plus the subnormal step) of the input, per block.
    xh, xd = make((256, 2048), "f32", seed=11, specials=False)
    q, s = H.hq_quantize_fp8_blockwise(xd, O.E4M3, 128)
    r = host(H.hq_dequantize_fp8_blockwise(q, s, O.E4M3, 128))
    torch.cuda.synchronize()
    sc = np.repeat(host(s), 128, axis=1)
    err = np.abs(r.astype(np.float64) - xh)
    assert (err <= np.abs(xh) * (2.0 ** -4 + 2.0 ** -20) + sc * 2.0 ** -10).all()


def test_blockwise_full_size_sweep_input():
    xb = W.sweep()
    rows, cols = xb.shape
    q, s = H.hq_quantize_fp8_blockwise(dev_bf16(xb), O.E4M3, 128)
    torch.cuda.synchronize()
    # sampled rows, checked one by one against the oracle
    rng = np.random.default_rng(1)
    for r in rng.choice(rows, 24, replace=False):
        qo, so, _ = O.quantize_blockwise(xb[r:r + 1], O.E4M3, 128)
        np.testing.assert_array_equal(host(q[r:r + 1]), qo)
        np.testing.assert_array_equal(host(s[r:r + 1]).view(np.uint32), so.view(np.uint32))
    H.hq_check_device_error()
