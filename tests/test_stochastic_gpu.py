"""GPU parity of the stochastic E5M2 quantize (hip-quant README "Stochastic
E5M2 Backward Gradients") against the oracle, through the C ABI: codes,
dequant scales and amax bit-exact for every granularity and input type, the
draws reproducible by seed, the workspace zero again after each call.

Inputs mix a wide dynamic range so that many scaled values fall in E5M2's
subnormal range (steps of 2^-16), plus NaN, +-Inf, -0 and f32 subnormals.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from fp8_dynamic_quantization_amax_b200 import _hq as H
from _gpu import dev_bf16, host

pytestmark = pytest.mark.gpu
SHAPES = [(1, 16), (7, 40), (33, 264), (130, 1024), (5, 8200)]


def make(shape, dtype, seed):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal(shape) * np.exp(rng.uniform(-12, 4, shape))).astype(np.float32)
    flat = x.reshape(-1)
    if flat.size >= 16:
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
@pytest.mark.parametrize("gran", [O.PER_TENSOR, O.PER_TOKEN, O.PER_CHANNEL])
def test_stochastic_e5m2_bit_exact(dtype, gran):
    for i, shape in enumerate(SHAPES):
        xh, xd = make(shape, dtype, seed=800 + 10 * i + gran)
        rows, cols = shape
        seed = (0x9E3779B97F4A7C15 * (i + 1)) & ((1 << 64) - 1)
        ns = H.hq_scale_count(gran, rows, cols)
        ws = torch.zeros(max(H.hq_quantize_workspace_bytes(gran, rows, cols, False), 256), dtype=torch.uint8,
                         device="cuda")
        a = torch.full((ns,), -1.0, device="cuda")
        q, s = H.hq_quantize_e5m2_stochastic(xd, gran, seed=seed, amax_out=a, workspace=ws)
        torch.cuda.synchronize()
        qo, so, ao = O.quantize_e5m2_sr(xh, gran, seed)
        np.testing.assert_array_equal(host(q), qo, err_msg="codes %s %s gran %d" % (shape, dtype, gran))
        np.testing.assert_array_equal(host(s).view(np.uint32), so.view(np.uint32))
        np.testing.assert_array_equal(host(a).view(np.uint32), ao.view(np.uint32))
        assert (host(ws) == 0).all()
    H.hq_check_device_error()


def test_stochastic_reproducible_by_seed():
    xh, xd = make((64, 512), "bf16", seed=3)
    q1, _ = H.hq_quantize_e5m2_stochastic(xd, O.PER_TOKEN, seed=42)
    q2, _ = H.hq_quantize_e5m2_stochastic(xd, O.PER_TOKEN, seed=42)
    q3, _ = H.hq_quantize_e5m2_stochastic(xd, O.PER_TOKEN, seed=43)
    torch.cuda.synchronize()
    assert torch.equal(q1, q2) and not torch.equal(q1, q3)


def test_stochastic_full_size_sweep_input():
    xb = W.sweep()
    q, s = H.hq_quantize_e5m2_stochastic(dev_bf16(xb), O.PER_TENSOR, seed=2024)
    torch.cuda.synchronize()
    qo, so, _ = O.quantize_e5m2_sr(xb, O.PER_TENSOR, 2024)
    assert np.array_equal(host(q), qo)
    assert host(s).view(np.uint32)[0] == so.view(np.uint32)[0]
    H.hq_check_device_error()
