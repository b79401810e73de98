"""hq_quantize_fp8_noalloc, through the C ABI.

This entry point serves callers that cannot allocate device memory: they hand
over only their input and output buffers, so the per-tensor, per-channel and
delayed modes take their scratch from a static device array inside the
library instead of a caller workspace.  These tests check that it gives the
same codes, dequant scales, amax and ring updates as hq_quantize_fp8 with a
caller workspace (the quantize tolerance is bit-exact), on two calls in a
row.  They also check that a shape too large for the array is refused before
any launch, leaving the outputs untouched, and that the array is left clean
for the next call.

The file is named so that pytest collects it last; it also passes on its
own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W
from fp8_dynamic_quantization_amax_b200 import _hq as H

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def noalloc_call(x, fmt, gran, ring=None, idx=0, margin=0):
    rows, cols = x.shape
    ns = H.hq_scale_count(gran, rows, cols)
    q = torch.full((rows, cols), 0xAB, dtype=torch.uint8, device="cuda")
    s = torch.full((ns,), -3.0, dtype=torch.float32, device="cuda")
    a = torch.full((ns,), -3.0, dtype=torch.float32, device="cuda")
    ring_len = 0 if ring is None else ring.numel() - 2
    st = H.lib.hq_quantize_fp8_noalloc(_p(x), H._DT[x.dtype], rows, cols, fmt, gran, _p(q), _p(s), _p(a),
                                       _p(ring), ring_len, idx, margin,
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, q, s, a


def workspace_call(x, fmt, gran, ring=None, idx=0, margin=0):
    rows, cols = x.shape
    ns = H.hq_scale_count(gran, rows, cols)
    ws = torch.zeros(max(H.hq_quantize_workspace_bytes(gran, rows, cols, ring is not None), 256),
                     dtype=torch.uint8, device="cuda")
    a = torch.empty((ns,), dtype=torch.float32, device="cuda")
    q, s = H.hq_quantize_fp8(x, fmt, gran, amax_out=a, ring=ring, ring_idx=idx, ring_margin=margin, workspace=ws)
    return q, s, a


def _input(shape, dtype, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(shape).astype(np.float32) * np.float32(5.0)
    x.reshape(-1)[:3] = [np.nan, np.inf, -0.0]
    if dtype == torch.bfloat16:
        return torch.from_numpy(W.f32_to_bf16_bits(x).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(x).to(dtype).cuda()


def _same(t1, t2):
    return torch.equal(t1.view(torch.uint8) if t1.dtype == torch.uint8 else t1.view(torch.int32),
                       t2.view(torch.uint8) if t2.dtype == torch.uint8 else t2.view(torch.int32))


@pytest.mark.parametrize("gran,shape,dtype", [
    (H.PER_TENSOR, (300, 520), torch.bfloat16),
    (H.PER_CHANNEL, (257, 4104), torch.bfloat16),
    (H.PER_CHANNEL, (9, 32764), torch.float16),      # the largest per-channel width that fits
    (H.PER_TOKEN, (33, 1000), torch.float32),        # needs no scratch at all
])
@pytest.mark.parametrize("fmt", [H.E4M3, H.E5M2])
def test_noalloc_matches_workspace_entry_point_twice(gran, shape, dtype, fmt):
    x = _input(shape, dtype, seed=shape[1] + fmt)
    q_ref, s_ref, a_ref = workspace_call(x, fmt, gran)
    for _ in range(2):  # two calls in a row share the static scratch
        st, q, s, a = noalloc_call(x, fmt, gran)
        assert st == H.HQ_OK, H.lib.hq_last_error().decode()
        torch.cuda.synchronize()
        assert _same(q, q_ref) and _same(s, s_ref) and _same(a, a_ref)
    H.hq_check_device_error()


@pytest.mark.parametrize("gran,shape,dtype", [
    (H.PER_TENSOR, (2048, 4096), torch.bfloat16),    # 16 MiB: the single-launch per-tensor kernel
    (H.PER_CHANNEL, (256, 32760), torch.bfloat16),   # 16 MiB, 16 column strips: the single-launch per-channel kernel
    (H.PER_CHANNEL, (128, 8192), torch.float32),     # exactly 4 MiB
])
def test_noalloc_single_launch_kernels_twice_vs_oracle(gran, shape, dtype):
    # Inputs of 4 MiB and more take the single-launch kernels, whose grid
    # barrier counters and departure count live in the scratch and must be
    # back at zero for the next call.
    import oracle as O
    x = _input(shape, dtype, seed=11 + shape[0])
    xh = x.view(torch.int16).cpu().numpy().view(np.uint16) if dtype == torch.bfloat16 else x.cpu().numpy()
    q_o, s_o, a_o = O.quantize(xh, O.E4M3, gran)
    q_ref, s_ref, a_ref = workspace_call(x, H.E4M3, gran)
    torch.cuda.synchronize()
    for _ in range(2):
        st, q, s, a = noalloc_call(x, H.E4M3, gran)
        assert st == H.HQ_OK, H.lib.hq_last_error().decode()
        torch.cuda.synchronize()
        assert _same(q, q_ref) and _same(s, s_ref) and _same(a, a_ref)
        np.testing.assert_array_equal(q.cpu().numpy(), q_o)
        np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), s_o.view(np.uint32))
        np.testing.assert_array_equal(a.cpu().numpy().view(np.uint32), a_o.view(np.uint32))
    H.hq_check_device_error()


def test_noalloc_delayed_ring_two_steps():
    L = 16
    ring_a = torch.zeros(L + 2, dtype=torch.float32, device="cuda")
    ring_a[L] = 1.0
    ring_b = ring_a.clone()
    for step in range(2):
        x = _input((64, 1000), torch.float32, seed=70 + step)
        q_ref, s_ref, a_ref = workspace_call(x, H.E4M3, H.PER_TENSOR, ring=ring_a, idx=step)
        st, q, s, a = noalloc_call(x, H.E4M3, H.PER_TENSOR, ring=ring_b, idx=step)
        assert st == H.HQ_OK, H.lib.hq_last_error().decode()
        torch.cuda.synchronize()
        assert _same(q, q_ref) and _same(s, s_ref) and _same(a, a_ref)
        assert _same(ring_b, ring_a)
    H.hq_check_device_error()


def test_noalloc_checks_arguments_before_the_size_limit():
    # an invalid granularity with a shape the scratch could not hold: the
    # argument error comes first, as hq_quantize_fp8 would report it
    x = _input((4, 40000), torch.bfloat16, seed=5)
    st, q, s, a = noalloc_call(x, H.E4M3, H.PER_TENSOR)
    assert st == H.HQ_OK
    bad = H.lib.hq_quantize_fp8_noalloc(_p(x), H._DT[x.dtype], 4, 40000, H.E4M3, 7, _p(q), _p(s), _p(a),
                                        None, 0, 0, 0, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert bad == 1  # HQ_ERR_INVALID_ARG
    assert "granularity" in H.lib.hq_last_error().decode()


def test_noalloc_refuses_a_shape_beyond_its_scratch():
    x = _input((4, 40000), torch.bfloat16, seed=3)   # per-channel needs > 256 KiB here
    st, q, s, a = noalloc_call(x, H.E4M3, H.PER_CHANNEL)
    assert st == 8  # HQ_ERR_TOO_LARGE
    assert "scratch" in H.lib.hq_last_error().decode()
    torch.cuda.synchronize()
    assert (q == 0xAB).all() and (s == -3.0).all()
    # the next call that fits still works and is exact
    y = _input((40, 300), torch.bfloat16, seed=4)
    q_ref, s_ref, _ = workspace_call(y, H.E4M3, H.PER_CHANNEL)
    st, q, s, _ = noalloc_call(y, H.E4M3, H.PER_CHANNEL)
    assert st == H.HQ_OK
    torch.cuda.synchronize()
    assert _same(q, q_ref) and _same(s, s_ref)
