"""CPU oracle for dynamic FP8 quantization and the scaled FP8 GEMM.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
benchmark's CPU-baseline / reference legs, never by the product package.
It is a thin ctypes layer over hq_oracle.c (plain C, single-threaded); all
arithmetic is in that file.  It shares nothing with the CUDA library.

Every function here cites the page passage it follows in hq_oracle.c.
"""
import ctypes
import os

import numpy as np

from . import build as _build

E4M3, E5M2 = 0, 1
F32, BF16, F16 = 0, 1, 2
PER_TENSOR, PER_TOKEN, PER_CHANNEL = 0, 1, 2

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        i32 = ctypes.c_int32
        ci = ctypes.c_int
        L.hqo_decode.argtypes = [ctypes.c_uint8, ci]
        L.hqo_decode.restype = ctypes.c_double
        L.hqo_encode_sat.argtypes = [ctypes.c_float, ci]
        L.hqo_encode_sat.restype = ctypes.c_uint8
        L.hqo_fmax.argtypes = [ci]
        L.hqo_fmax.restype = ctypes.c_double
        L.hqo_multiplier.argtypes = [ctypes.c_float, ci]
        L.hqo_multiplier.restype = ctypes.c_float
        L.hqo_scale_count.argtypes = [ci, i64, i64]
        L.hqo_scale_count.restype = i64
        L.hqo_double_to_bf16.argtypes = [ctypes.c_double]
        L.hqo_double_to_bf16.restype = ctypes.c_uint16
        L.hqo_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.hqo_bf16_to_f32.restype = ctypes.c_float
        L.hqo_amax.argtypes = [P, ci, i64, i64, ci, P]
        L.hqo_amax.restype = None
        L.hqo_quantize.argtypes = [P, ci, i64, i64, ci, ci, P, P, P, P, ci, ci, ci]
        L.hqo_quantize.restype = ci
        L.hqo_gemm_a8w8.argtypes = [P, P, ci, P, i64, P, i64, i64, i64, i64, P, P]
        L.hqo_gemm_a8w8.restype = None
        L.hqo_splitmix64_next.argtypes = [P]
        L.hqo_splitmix64_next.restype = ctypes.c_uint64
        L.hqo_sr_bits.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        L.hqo_sr_bits.restype = ctypes.c_uint32
        L.hqo_encode_e5m2_sr.argtypes = [ctypes.c_float, ctypes.c_uint32]
        L.hqo_encode_e5m2_sr.restype = ctypes.c_uint8
        L.hqo_quantize_e5m2_sr.argtypes = [P, ci, i64, i64, ci, ctypes.c_uint64, P, P, P]
        L.hqo_quantize_e5m2_sr.restype = ci
        L.hqo_quantize_blockwise.argtypes = [P, ci, i64, i64, ci, i64, ci, ctypes.c_uint64, P, P, P]
        L.hqo_quantize_blockwise.restype = ci
        L.hqo_dequantize_blockwise.argtypes = [P, ci, i64, i64, i64, P, ci, P]
        L.hqo_dequantize_blockwise.restype = ci
        L.hqo_gemm_a8w8_bias.argtypes = [P, P, ci, P, i64, P, i64, P, i64, i64, i64, P]
        L.hqo_gemm_a8w8_bias.restype = None
        L.hqo_gemm_blockscaled.argtypes = [P, P, ci, P, P, i64, P, i64, i64, i64, P, P]
        L.hqo_gemm_blockscaled.restype = None
        L.hqo_gemm_blockscaled_entries.argtypes = [P, P, ci, P, P, i64, P, i64, P, P, i64, P]
        L.hqo_gemm_blockscaled_entries.restype = None
        L.hqo_gemm_a8w8_entries.argtypes = [P, P, ci, P, i64, P, i64, i64, P, P, i64, P]
        L.hqo_gemm_a8w8_entries.restype = None
        L.hqo_grouped_gemm_a8w8.argtypes = [P, P, ci, P, P, P, i32, i64, i64, i64, P]
        L.hqo_grouped_gemm_a8w8.restype = ci
        L.hqo_grouped_gemm_bf16.argtypes = [P, P, P, i32, i64, i64, i64, P]
        L.hqo_grouped_gemm_bf16.restype = ci
        L.hqo_encode_sat_array.argtypes = [P, i64, ci, P]
        L.hqo_encode_sat_array.restype = None
        L.hqo_decode_array.argtypes = [P, i64, ci, P]
        L.hqo_decode_array.restype = None
        L.hqo_ring_update.argtypes = [ctypes.c_float, ci, P, ci, ci, ci]
        L.hqo_ring_update.restype = None
        L.hqo_double_to_f16.argtypes = [ctypes.c_double]
        L.hqo_double_to_f16.restype = ctypes.c_uint16
        L.hqo_grad_bias.argtypes = [P, ci, i64, i64, P, P]
        L.hqo_grad_bias.restype = None
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(x):
    if x.dtype == np.float32:
        return F32
    if x.dtype == np.uint16:
        return BF16  # bf16 carried as raw uint16 bit patterns
    if x.dtype == np.float16:
        return F16
    raise TypeError("oracle inputs are float32, float16 or bf16 bit patterns (uint16)")


def decode(code: int, fmt: int) -> float:
    return lib().hqo_decode(code, fmt)


def encode_sat(y: float, fmt: int) -> int:
    return lib().hqo_encode_sat(y, fmt)


def encode_sat_array(y: np.ndarray, fmt: int) -> np.ndarray:
    y = np.ascontiguousarray(y, np.float32).reshape(-1)
    out = np.empty(y.size, np.uint8)
    lib().hqo_encode_sat_array(_p(y), y.size, fmt, _p(out))
    return out


def decode_array(c: np.ndarray, fmt: int) -> np.ndarray:
    c = np.ascontiguousarray(c, np.uint8).reshape(-1)
    out = np.empty(c.size, np.float64)
    lib().hqo_decode_array(_p(c), c.size, fmt, _p(out))
    return out


def fmax(fmt: int) -> float:
    return lib().hqo_fmax(fmt)


def multiplier(amax: float, fmt: int) -> float:
    return lib().hqo_multiplier(amax, fmt)


def scale_count(gran: int, rows: int, cols: int) -> int:
    return lib().hqo_scale_count(gran, rows, cols)


def double_to_bf16(v: float) -> int:
    return lib().hqo_double_to_bf16(v)


def amax(x: np.ndarray, gran: int) -> np.ndarray:
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    out = np.zeros(scale_count(gran, rows, cols), np.float32)
    lib().hqo_amax(_p(x), _dtype_code(x), rows, cols, gran, _p(out))
    return out


def quantize(x: np.ndarray, fmt: int, gran: int, ring: np.ndarray = None,
             ring_idx: int = 0, ring_margin: int = 0):
    """Returns (codes uint8 [rows, cols], dequant scales f32, amax f32).

    With `ring` (float32 [len+2], updated in place) this is the delayed
    per-tensor mode."""
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    n = scale_count(gran, rows, cols)
    q = np.empty((rows, cols), np.uint8)
    scales = np.empty(max(n, 1), np.float32)[:n]
    am = np.empty(max(n, 1), np.float32)[:n]
    ring_len = 0
    if ring is not None:
        assert ring.dtype == np.float32 and ring.flags.c_contiguous
        ring_len = ring.size - 2
    rc = lib().hqo_quantize(_p(x), _dtype_code(x), rows, cols, fmt, gran, _p(q),
                            _p(scales), _p(am), _p(ring), ring_len, ring_idx, ring_margin)
    if rc != 0:
        raise ValueError("oracle quantize: invalid arguments")
    return q, scales, am


def ring_update(amax_value: float, fmt: int, ring: np.ndarray, ring_idx: int, ring_margin: int = 0):
    """One delayed-scaling ring step (in place) given this step's amax."""
    assert ring.dtype == np.float32 and ring.flags.c_contiguous
    lib().hqo_ring_update(amax_value, fmt, _p(ring), ring.size - 2, ring_idx, ring_margin)


def gemm_a8w8(xq, wq, fmt, x_scale, w_scale, return_ref=False):
    xq = np.ascontiguousarray(xq, np.uint8)
    wq = np.ascontiguousarray(wq, np.uint8)
    xs = np.ascontiguousarray(x_scale, np.float32).reshape(-1)
    ws = np.ascontiguousarray(w_scale, np.float32).reshape(-1)
    M, K = xq.shape
    N = wq.shape[0]
    out = np.empty((M, N), np.uint16)
    ref = np.empty((M, N), np.float64) if return_ref else None
    lib().hqo_gemm_a8w8(_p(xq), _p(wq), fmt, _p(xs), xs.size, _p(ws), ws.size,
                        M, N, K, _p(out), _p(ref))
    return (out, ref) if return_ref else out


def splitmix64_outputs(seed, count):
    """The first `count` outputs of a SplitMix64 generator started at `seed`."""
    st = ctypes.c_uint64(seed)
    return [lib().hqo_splitmix64_next(ctypes.byref(st)) for _ in range(count)]


def sr_bits(seed, idx):
    """The 32-bit draw of element index `idx` under `seed` (stochastic rounding)."""
    return lib().hqo_sr_bits(seed, idx)


def encode_e5m2_sr(y, u):
    """E5M2 code of the f32 value y rounded stochastically with draw u."""
    return lib().hqo_encode_e5m2_sr(float(np.float32(y)), int(u))


def quantize_e5m2_sr(x, gran, seed):
    """Dynamic E5M2 quantize with stochastic rounding: (codes, dequant scales,
    amax); amax and scales as quantize(), the draws by flat element index."""
    x = np.ascontiguousarray(x)
    dt = _dtype_code(x)
    rows, cols = x.shape
    ns = lib().hqo_scale_count(gran, rows, cols)
    q = np.empty((rows, cols), np.uint8)
    s = np.empty(max(ns, 1), np.float32)[:ns]
    a = np.empty(max(ns, 1), np.float32)[:ns]
    rc = lib().hqo_quantize_e5m2_sr(_p(x), dt, rows, cols, gran, seed, _p(q), _p(s), _p(a))
    if rc != 0:
        raise ValueError("invalid arguments")
    return q, s, a


def quantize_blockwise(x, fmt, block, stochastic=False, seed=0):
    """Block-wise quantize along the last dimension: (codes [rows, cols],
    dequant scales f32 [rows, ceil(cols/block)], amax of the same shape)."""
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    nb = -(-cols // block)
    q = np.empty((rows, cols), np.uint8)
    s = np.empty((rows, nb), np.float32)
    a = np.empty((rows, nb), np.float32)
    rc = lib().hqo_quantize_blockwise(_p(x), _dtype_code(x), rows, cols, fmt, block, 1 if stochastic else 0, seed,
                                      _p(q), _p(s), _p(a))
    if rc != 0:
        raise ValueError("invalid arguments")
    return q, s, a


def dequantize_blockwise(q, fmt, block, scales, bf16=False):
    """f32(dec(q) * block scale), or its bf16 bits."""
    q = np.ascontiguousarray(q, np.uint8)
    sc = np.ascontiguousarray(scales, np.float32)
    rows, cols = q.shape
    out = np.empty((rows, cols), np.uint16 if bf16 else np.float32)
    rc = lib().hqo_dequantize_blockwise(_p(q), fmt, rows, cols, block, _p(sc), 1 if bf16 else 0, _p(out))
    if rc != 0:
        raise ValueError("invalid arguments")
    return out


def gemm_a8w8_bias(xq, wq, fmt, x_scale, w_scale, bias_bf16_bits):
    """bf16 bits of x_scale * w_scale * (XQ . WQ^T) + bias, rounded once."""
    xq = np.ascontiguousarray(xq, np.uint8)
    wq = np.ascontiguousarray(wq, np.uint8)
    xs = np.ascontiguousarray(x_scale, np.float32).reshape(-1)
    ws = np.ascontiguousarray(w_scale, np.float32).reshape(-1)
    b = np.ascontiguousarray(bias_bf16_bits, np.uint16).reshape(-1)
    M, K = xq.shape
    N = wq.shape[0]
    assert b.size == N
    out = np.empty((M, N), np.uint16)
    lib().hqo_gemm_a8w8_bias(_p(xq), _p(wq), fmt, _p(xs), xs.size, _p(ws), ws.size, _p(b), M, N, K, _p(out))
    return out


def gemm_blockscaled(xq, wq, fmt, x_scales, w_scales, block, bias_bf16_bits=None, return_ref=False):
    """bf16 bits of sum_b xs[m,b] ws[n,b] S_b[m,n] (+ bias[n]), one rounding;
    x_scales [M, ceil(K/block)], w_scales [N, ceil(K/block)]."""
    xq = np.ascontiguousarray(xq, np.uint8)
    wq = np.ascontiguousarray(wq, np.uint8)
    M, K = xq.shape
    N = wq.shape[0]
    nb = -(-K // block)
    xs = np.ascontiguousarray(x_scales, np.float32).reshape(M, nb)
    ws = np.ascontiguousarray(w_scales, np.float32).reshape(N, nb)
    b = None if bias_bf16_bits is None else np.ascontiguousarray(bias_bf16_bits, np.uint16).reshape(N)
    out = np.empty((M, N), np.uint16)
    ref = np.empty((M, N), np.float64) if return_ref else None
    lib().hqo_gemm_blockscaled(_p(xq), _p(wq), fmt, _p(xs), _p(ws), block, _p(b), M, N, K, _p(out), _p(ref))
    return (out, ref) if return_ref else out


def gemm_blockscaled_entries(xq, wq, fmt, x_scales, w_scales, block, ms, ns, bias_bf16_bits=None):
    xq = np.ascontiguousarray(xq, np.uint8)
    wq = np.ascontiguousarray(wq, np.uint8)
    K = xq.shape[1]
    xs = np.ascontiguousarray(x_scales, np.float32)
    ws = np.ascontiguousarray(w_scales, np.float32)
    b = None if bias_bf16_bits is None else np.ascontiguousarray(bias_bf16_bits, np.uint16)
    ms = np.ascontiguousarray(ms, np.int64)
    ns = np.ascontiguousarray(ns, np.int64)
    out = np.empty(ms.size, np.uint16)
    lib().hqo_gemm_blockscaled_entries(_p(xq), _p(wq), fmt, _p(xs), _p(ws), block, _p(b), K, _p(ms), _p(ns),
                                       ms.size, _p(out))
    return out


def gemm_a8w8_entries(xq, wq, fmt, x_scale, w_scale, ms, ns):
    xq = np.ascontiguousarray(xq, np.uint8)
    wq = np.ascontiguousarray(wq, np.uint8)
    xs = np.ascontiguousarray(x_scale, np.float32).reshape(-1)
    ws = np.ascontiguousarray(w_scale, np.float32).reshape(-1)
    ms = np.ascontiguousarray(ms, np.int64)
    ns = np.ascontiguousarray(ns, np.int64)
    K = xq.shape[1]
    out = np.empty(ms.size, np.uint16)
    lib().hqo_gemm_a8w8_entries(_p(xq), _p(wq), fmt, _p(xs), xs.size, _p(ws), ws.size,
                                K, _p(ms), _p(ns), ms.size, _p(out))
    return out


def grouped_gemm_a8w8(xq, wq, fmt, x_scale, w_scale, offsets, out=None):
    xq = np.ascontiguousarray(xq, np.uint8)
    wq = np.ascontiguousarray(wq, np.uint8)
    xs = np.ascontiguousarray(x_scale, np.float32).reshape(-1)
    ws = np.ascontiguousarray(w_scale, np.float32).reshape(-1)
    off = np.ascontiguousarray(offsets, np.int32)
    M, K = xq.shape
    E, N, _ = wq.shape
    if out is None:
        out = np.zeros((M, N), np.uint16)
    rc = lib().hqo_grouped_gemm_a8w8(_p(xq), _p(wq), fmt, _p(xs), _p(ws), _p(off),
                                     E, M, N, K, _p(out))
    if rc != 0:
        raise ValueError("oracle grouped gemm: malformed offsets")
    return out


def grouped_gemm_bf16(x, w, offsets, out=None):
    x = np.ascontiguousarray(x, np.uint16)
    w = np.ascontiguousarray(w, np.uint16)
    off = np.ascontiguousarray(offsets, np.int32)
    M, K = x.shape
    E, N, _ = w.shape
    if out is None:
        out = np.zeros((M, N), np.uint16)
    rc = lib().hqo_grouped_gemm_bf16(_p(x), _p(w), _p(off), E, M, N, K, _p(out))
    if rc != 0:
        raise ValueError("oracle grouped gemm: malformed offsets")
    return out


def double_to_f16(v: float) -> int:
    return lib().hqo_double_to_f16(v)


def grad_bias(g: np.ndarray, return_ref: bool = False):
    """Bias gradient: column sums of g [rows, cols] (fp64, rows in order),
    rounded once to g's dtype (bf16 bit patterns, float16 or float32)."""
    g = np.ascontiguousarray(g)
    rows, cols = g.shape
    dt = _dtype_code(g)
    out = np.empty(cols, {F32: np.float32, BF16: np.uint16, F16: np.float16}[dt])
    ref = np.empty(cols, np.float64) if return_ref else None
    lib().hqo_grad_bias(_p(g), dt, rows, cols, _p(out), _p(ref))
    return (out, ref) if return_ref else out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)
