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


# ------------------------------------------------------------ bias gradient
# AstrAI ops.cu linear_backward_fp8: grad_bias = g summed over dim 0, in g's
# dtype.  The GPU sums in f32 in a fixed order, the oracle in fp64; the
# tolerance is the f32 summation bound (rows * 2^-24 * sum |g|, doubled for
# the two levels of the kernel's sum) plus one step of the output dtype at
# the result (a value near a rounding boundary may round either way).
GB_SHAPES = [  # (rows, cols, dtype): vector and element paths, ragged strips and bands, one band and many
    (1, 8, "bf16"), (7, 24, "f16"), (300, 1001, "f32"), (1000, 2056, "bf16"), (130, 36, "f16"),
    (129, 4100, "f32"), (5000, 520, "bf16"), (9000, 264, "f16"), (0, 40, "bf16"),
]


def _as_f64(a, dtype):
    if dtype == "bf16":
        return O.bf16_bits_to_f32(a).astype(np.float64)
    return np.asarray(a).astype(np.float64)


def _step(v, dtype):
    mant = {"bf16": 7, "f16": 10, "f32": 23}[dtype]
    low = {"bf16": -133, "f16": -24, "f32": -149}[dtype]
    e = np.floor(np.log2(np.maximum(np.abs(v), 1e-300)))
    return np.maximum(2.0 ** (e - mant), 2.0 ** low)


def _abs_col_sums(gh, dtype):
    out = np.zeros(gh.shape[1], np.float64)
    for i in range(0, gh.shape[0], 1024):  # in row chunks: the full-size g would not fit as fp64
        v = _as_f64(gh[i:i + 1024], dtype)
        out += np.abs(np.where(np.isfinite(v), v, 0.0)).sum(axis=0)
    return out


def _check_grad_bias(got, gh, dtype):
    """got: the GPU result as bf16 bit patterns, f16 or f32 values."""
    want, ref = O.grad_bias(gh, return_ref=True)
    rows = gh.shape[0]
    got64, want64 = _as_f64(got, dtype), _as_f64(want, dtype)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got64), nan)
    inf = np.isinf(ref)
    assert np.array_equal(got64[inf], ref[inf])
    fin = ~(nan | inf)
    bound = 2.0 * rows * 2.0 ** -24 * _abs_col_sums(gh, dtype)[fin]
    err = np.abs(got64[fin] - ref[fin])
    assert (err <= bound + _step(ref[fin], dtype)).all(), np.max(err - bound - _step(ref[fin], dtype))
    # and never further than one output step from the oracle's own rounding
    assert (np.abs(got64[fin] - want64[fin]) <= _step(want64[fin], dtype) + bound).all()


def _fetch(t, dtype):
    return host_bits(t) if dtype == "bf16" else host(t)


@pytest.mark.parametrize("case", range(len(GB_SHAPES)))
def test_grad_bias_vs_oracle(case):
    rows, cols, dtype = GB_SHAPES[case]
    gh, gd = make((rows, cols), dtype, seed=600 + case, specials=rows * cols >= 5000)
    ws = torch.zeros(H.hq_grad_bias_workspace_bytes(rows, cols), dtype=torch.uint8, device="cuda")
    got = [H.hq_grad_bias(gd, workspace=ws) for _ in range(2)]
    torch.cuda.synchronize()
    a, b = _fetch(got[0], dtype), _fetch(got[1], dtype)
    assert np.array_equal(a.view(np.uint8), b.view(np.uint8))  # fixed order: identical bits
    _check_grad_bias(a, gh, dtype)
    assert (host(ws)[:256] == 0).all()  # the strip counters are back to zero
    H.hq_check_device_error()


def test_grad_bias_unaligned_rows_and_view():
    # g a view whose rows start off the 16-byte grid: the element path
    rows, cols = 777, 1029
    gh, gd = make((rows, cols + 3), "bf16", seed=650, specials=False)
    view = gd[:, 3:]  # not contiguous; the binding makes it contiguous
    got = H.hq_grad_bias(view)
    torch.cuda.synchronize()
    _check_grad_bias(host_bits(got), np.ascontiguousarray(gh[:, 3:]), "bf16")


def test_grad_bias_full_backward_shape():
    # g of the large layer's backward ([16384, 28672] bf16, ~N(0, 1)):
    # every column against the oracle
    rows, cols = 16384, 28672
    rng = np.random.default_rng(660)
    gh = W.f32_to_bf16_bits(rng.standard_normal((rows, cols), dtype=np.float32))
    got = H.hq_grad_bias(dev_bf16(gh))
    torch.cuda.synchronize()
    _check_grad_bias(host_bits(got), gh, "bf16")
    H.hq_check_device_error()
