"""ctypes binding of libhq.so (include/hq.h).

Argument marshalling only: every step of the path runs in the library's
CUDA kernels.  torch provides device memory and the current stream.  If the
library is missing this module raises at import time: there is no fallback.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhq.so")

HQ_OK = 0
STATUS_NAMES = {0: "HQ_OK", 1: "HQ_ERR_INVALID_ARG", 2: "HQ_ERR_MISALIGNED", 3: "HQ_ERR_OVERLAP",
                4: "HQ_ERR_WRONG_DEVICE", 5: "HQ_ERR_UNSUPPORTED_ARCH", 6: "HQ_ERR_CUDA",
                7: "HQ_ERR_TIMEOUT", 8: "HQ_ERR_TOO_LARGE"}
E4M3, E5M2 = 0, 1
PER_TENSOR, PER_TOKEN, PER_CHANNEL = 0, 1, 2
F32, BF16, F16 = 0, 1, 2

EXPORTED = ["hq_scale_count", "hq_granularity_name", "hq_scale_pair_name", "hq_quantize_workspace_bytes",
            "hq_quantize_fp8", "hq_quantize_fp8_transpose", "hq_quantize_e5m2_stochastic",
            "hq_quantize_fp8_blockwise", "hq_dequantize_fp8_blockwise", "hq_gemm_blockscaled",
            "hq_gemm_a8w8", "hq_gemm_a8w8_ex", "hq_gemm_a8w8_blockq", "hq_grouped_gemm_a8w8", "hq_grouped_gemm_bf16",
            "hq_quantize_fp8_noalloc", "hq_quantize_fp8_delayed_batch", "hq_grad_bias",
            "hq_grad_bias_workspace_bytes", "hq_debug_bounded_wait",
            "hq_check_device_error", "hq_last_error", "hq_version"]
NOALLOC_SCRATCH_BYTES = 256 * 1024


class DelayedTensor(ctypes.Structure):
    """hq_delayed_tensor: one tensor of a batched delayed quantize."""
    _fields_ = [("x", ctypes.c_void_p), ("n", ctypes.c_int64), ("q", ctypes.c_void_p),
                ("scale", ctypes.c_void_p), ("amax_out", ctypes.c_void_p), ("ring", ctypes.c_void_p),
                ("ring_len", ctypes.c_int32), ("ring_idx", ctypes.c_int32), ("ring_margin", ctypes.c_int32),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t)]


class HQError(RuntimeError):
    def __init__(self, status, message):
        self.status = status
        self.status_name = STATUS_NAMES.get(status, str(status))
        super().__init__("%s: %s" % (self.status_name, message))


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("libhq.so is not built (python fp8_dynamic_quantization_amax_b200/build.py); "
                          "there is no CPU fallback")
    L = ctypes.CDLL(LIB_PATH)
    P, i64, i32, ci, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int, ctypes.c_size_t
    L.hq_scale_count.argtypes = [ci, i64, i64]
    L.hq_scale_count.restype = i64
    L.hq_granularity_name.argtypes = [ci]
    L.hq_granularity_name.restype = ctypes.c_char_p
    L.hq_scale_pair_name.argtypes = [ci, ci, ctypes.c_char_p, sz]
    L.hq_scale_pair_name.restype = ci
    L.hq_quantize_workspace_bytes.argtypes = [ci, i64, i64, ci]
    L.hq_quantize_workspace_bytes.restype = sz
    L.hq_quantize_fp8.argtypes = [P, ci, i64, i64, ci, ci, P, P, P, P, i32, i32, i32, P, sz, P]
    L.hq_quantize_fp8.restype = ci
    L.hq_quantize_fp8_noalloc.argtypes = [P, ci, i64, i64, ci, ci, P, P, P, P, i32, i32, i32, P]
    L.hq_quantize_fp8_noalloc.restype = ci
    L.hq_quantize_fp8_delayed_batch.argtypes = [ctypes.POINTER(DelayedTensor), i32, ci, ci, P]
    L.hq_quantize_fp8_delayed_batch.restype = ci
    L.hq_debug_bounded_wait.argtypes = [ctypes.c_uint64, P]
    L.hq_debug_bounded_wait.restype = ci
    L.hq_gemm_blockscaled.argtypes = [P, P, ci, P, P, i64, P, i64, i64, i64, P, P]
    L.hq_gemm_blockscaled.restype = ci
    L.hq_quantize_fp8_blockwise.argtypes = [P, ci, i64, i64, ci, i64, ci, ctypes.c_uint64, P, P, P, P]
    L.hq_quantize_fp8_blockwise.restype = ci
    L.hq_dequantize_fp8_blockwise.argtypes = [P, ci, i64, i64, i64, P, ci, P, P]
    L.hq_dequantize_fp8_blockwise.restype = ci
    L.hq_quantize_e5m2_stochastic.argtypes = [P, ci, i64, i64, ci, ctypes.c_uint64, P, P, P, P, sz, P]
    L.hq_quantize_e5m2_stochastic.restype = ci
    L.hq_quantize_fp8_transpose.argtypes = [P, ci, i64, i64, ci, P, P, P, P, P, P, i32, i32, i32, P, sz, P]
    L.hq_quantize_fp8_transpose.restype = ci
    L.hq_grad_bias_workspace_bytes.argtypes = [i64, i64]
    L.hq_grad_bias_workspace_bytes.restype = sz
    L.hq_grad_bias.argtypes = [P, ci, i64, i64, P, P, sz, P]
    L.hq_grad_bias.restype = ci
    L.hq_gemm_a8w8.argtypes = [P, P, ci, P, i64, P, i64, i64, i64, i64, P, P]
    L.hq_gemm_a8w8.restype = ci
    L.hq_gemm_a8w8_ex.argtypes = [P, P, ci, P, i64, P, i64, P, i64, i64, i64, P, P, ci, P, P, P, i32, i32, i32, P,
                                  sz, P]
    L.hq_gemm_a8w8_ex.restype = ci
    L.hq_gemm_a8w8_blockq.argtypes = [P, P, ci, P, i64, P, i64, P, i64, i64, i64, P, ci, i64, P, P]
    L.hq_gemm_a8w8_blockq.restype = ci
    L.hq_grouped_gemm_a8w8.argtypes = [P, P, ci, P, i64, P, i64, P, i32, i64, i64, i64, P, P]
    L.hq_grouped_gemm_a8w8.restype = ci
    L.hq_grouped_gemm_bf16.argtypes = [P, P, P, i32, i64, i64, i64, P, P]
    L.hq_grouped_gemm_bf16.restype = ci
    L.hq_check_device_error.argtypes = []
    L.hq_check_device_error.restype = ci
    L.hq_last_error.argtypes = []
    L.hq_last_error.restype = ctypes.c_char_p
    L.hq_version.argtypes = []
    L.hq_version.restype = ctypes.c_char_p
    return L


lib = _load()


def check(status):
    if status != HQ_OK:
        raise HQError(status, lib.hq_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


_DT = {torch.float32: F32, torch.bfloat16: BF16, torch.float16: F16}
_ws_cache = {}


def _workspace(device, nbytes, slot=0):
    """A zero-filled workspace per (device, size, slot).  The library returns
    its accumulator words to zero after each call, so calls that run one
    after another on one stream can share it; tensors of one batched call run
    at once and take different slots."""
    if nbytes == 0:
        return None
    key = (device, nbytes, slot)
    ws = _ws_cache.get(key)
    if ws is None:
        ws = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


def hq_scale_count(gran, rows, cols):
    return lib.hq_scale_count(gran, rows, cols)


def hq_granularity_name(gran):
    r = lib.hq_granularity_name(gran)
    return None if r is None else r.decode()


def hq_scale_pair_name(act, weight):
    buf = ctypes.create_string_buffer(64)
    n = lib.hq_scale_pair_name(act, weight, buf, 64)
    return None if n < 0 else buf.value.decode()


def hq_quantize_workspace_bytes(gran, rows, cols, delayed=False):
    return lib.hq_quantize_workspace_bytes(gran, rows, cols, 1 if delayed else 0)


def hq_quantize_fp8(x, fmt=E4M3, gran=PER_TOKEN, q=None, scales=None, amax_out=None, ring=None,
                    ring_idx=0, ring_margin=0, workspace=None, stream=None):
    """Quantize a 2-D CUDA tensor (f32 / bf16 / f16).  Returns (q uint8,
    dequant scales f32).  With `ring` (f32 [len+2]) this is the delayed
    per-tensor mode; the ring is updated in place on the device."""
    if x.dim() != 2:
        raise ValueError("x must be 2-D")
    if x.dtype not in _DT:
        raise ValueError("x must be float32, bfloat16 or float16")
    x = x.contiguous()
    rows, cols = x.shape
    ns = hq_scale_count(gran, rows, cols)
    if q is None:
        q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((max(ns, 0),), dtype=torch.float32, device=x.device)
    ring_len = 0
    if ring is not None:
        ring_len = ring.numel() - 2
    need = hq_quantize_workspace_bytes(gran, rows, cols, ring is not None)
    if workspace is None:
        workspace = _workspace(x.device, need)
    check(lib.hq_quantize_fp8(_ptr(x), _DT[x.dtype], rows, cols, fmt, gran, _ptr(q), _ptr(scales),
                              _ptr(amax_out), _ptr(ring), ring_len, ring_idx, ring_margin,
                              _ptr(workspace), 0 if workspace is None else workspace.numel(),
                              _stream(stream)))
    return q, scales


def hq_quantize_fp8_delayed_batch(items, fmt=E4M3, stream=None):
    """Delayed per-tensor quantize of up to 8 CUDA tensors of one dtype in one
    launch.  items: list of dicts with x (any shape, contiguous), ring (f32
    [len+2]), ring_idx, and optionally ring_margin, q, scale, amax_out,
    workspace.  Returns [(q, scale)] in order; each ring is stepped in place."""
    if not 1 <= len(items) <= 8:
        raise ValueError("1 to 8 tensors")
    dt = items[0]["x"].dtype
    if dt not in _DT or any(it["x"].dtype != dt for it in items):
        raise ValueError("all tensors must share one of float32, bfloat16, float16")
    arr = (DelayedTensor * len(items))()
    keep, outs = [], []
    for i, it in enumerate(items):
        x = it["x"].contiguous()
        n = x.numel()
        q = it.get("q")
        if q is None:
            q = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
        scale = it.get("scale")
        if scale is None:
            scale = torch.empty((1,), dtype=torch.float32, device=x.device)
        ring = it["ring"]
        ws = it.get("workspace")
        if ws is None:
            ws = _workspace(x.device, hq_quantize_workspace_bytes(PER_TENSOR, 1, n, True), slot=1 + i)
        am = it.get("amax_out")
        arr[i] = DelayedTensor(x.data_ptr(), n, q.data_ptr(), scale.data_ptr(), None if am is None else am.data_ptr(),
                               ring.data_ptr(), ring.numel() - 2, it["ring_idx"], it.get("ring_margin", 0),
                               None if ws is None else ws.data_ptr(), 0 if ws is None else ws.numel())
        keep += [x, ws]
        outs.append((q, scale))
    check(lib.hq_quantize_fp8_delayed_batch(arr, len(items), _DT[dt], fmt, _stream(stream)))
    return outs


def hq_quantize_fp8_blockwise(x, fmt=E4M3, block=32, stochastic=False, seed=0, amax_out=None, stream=None):
    """Block-wise quantize along the last dimension.  Returns (q uint8
    [rows, cols], dequant scales f32 [rows, ceil(cols / block)])."""
    if x.dim() != 2:
        raise ValueError("x must be 2-D")
    x = x.contiguous()
    rows, cols = x.shape
    q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    scales = torch.empty((rows, -(-cols // block)), dtype=torch.float32, device=x.device)
    check(lib.hq_quantize_fp8_blockwise(_ptr(x), _DT[x.dtype], rows, cols, fmt, block, 1 if stochastic else 0,
                                        seed & ((1 << 64) - 1), _ptr(q), _ptr(scales), _ptr(amax_out),
                                        _stream(stream)))
    return q, scales


def hq_gemm_blockscaled(xq, wq, x_scales, w_scales, fmt=E4M3, block=32, bias=None, out=None, stream=None):
    """bf16 [M, N] = sum over K blocks of x_scales[m,b] w_scales[n,b] (XQ . WQ^T
    over block b) (+ bias)."""
    M, K = xq.shape
    N = wq.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    check(lib.hq_gemm_blockscaled(_ptr(xq.contiguous()), _ptr(wq.contiguous()), fmt, _ptr(x_scales.contiguous()),
                                  _ptr(w_scales.contiguous()), block, _ptr(bias), M, N, K, _ptr(out),
                                  _stream(stream)))
    return out


def hq_linear_blockwise(x, w, bias=None, fmt=E4M3, block=32, out=None, stream=None):
    """The block-scaled linear on bf16 / f16 / f32 operands: x [M, K] and
    w [N, K] quantized block-wise along K (three C-ABI calls: two
    hq_quantize_fp8_blockwise, one hq_gemm_blockscaled).  Returns bf16
    out [M, N] = x . w^T (+ bias) within the FP8 error."""
    xq, xs = hq_quantize_fp8_blockwise(x, fmt, block, stream=stream)
    wq, ws = hq_quantize_fp8_blockwise(w, fmt, block, stream=stream)
    return hq_gemm_blockscaled(xq, wq, xs, ws, fmt, block, bias=bias, out=out, stream=stream)


def hq_dequantize_fp8_blockwise(q, scales, fmt=E4M3, block=32, out_dtype=torch.float32, stream=None):
    """f32(dec(q) * block scale), as float32 or rounded to bfloat16."""
    rows, cols = q.shape
    out = torch.empty((rows, cols), dtype=out_dtype, device=q.device)
    check(lib.hq_dequantize_fp8_blockwise(_ptr(q.contiguous()), fmt, rows, cols, block, _ptr(scales.contiguous()),
                                          _DT[out_dtype], _ptr(out), _stream(stream)))
    return out


def hq_quantize_e5m2_stochastic(x, gran=PER_TENSOR, seed=0, q=None, scales=None, amax_out=None, workspace=None,
                                stream=None):
    """Dynamic E5M2 quantize with stochastic rounding (seeded, reproducible).
    Returns (q uint8, dequant scales f32)."""
    if x.dim() != 2:
        raise ValueError("x must be 2-D")
    x = x.contiguous()
    rows, cols = x.shape
    ns = hq_scale_count(gran, rows, cols)
    if q is None:
        q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((max(ns, 0),), dtype=torch.float32, device=x.device)
    need = hq_quantize_workspace_bytes(gran, rows, cols, False)
    if workspace is None and need > 0:
        workspace = _workspace(x.device, need)
    check(lib.hq_quantize_e5m2_stochastic(_ptr(x), _DT[x.dtype], rows, cols, gran, seed & ((1 << 64) - 1), _ptr(q),
                                          _ptr(scales), _ptr(amax_out), _ptr(workspace),
                                          0 if workspace is None else workspace.numel(), _stream(stream)))
    return q, scales


def hq_quantize_fp8_transpose(x, fmt=E4M3, q=False, multiplier=None, amax_out=None, ring=None, ring_idx=0,
                              ring_margin=0, workspace=None, stream=None):
    """Per-tensor quantize of a 2-D CUDA tensor writing the codes transposed
    (qt [cols, rows]) and, with q=True, also row-major.  The multiplier is the
    ring's (delayed, the ring stepped), a caller's device f32 `multiplier`
    (static), or the tensor's own fmax/amax (dynamic).  Returns (q or None,
    qt, dequant scale f32[1])."""
    if x.dim() != 2:
        raise ValueError("x must be 2-D")
    x = x.contiguous()
    rows, cols = x.shape
    qo = torch.empty((rows, cols), dtype=torch.uint8, device=x.device) if q else None
    qt = torch.empty((cols, rows), dtype=torch.uint8, device=x.device)
    scales = torch.empty((1,), dtype=torch.float32, device=x.device)
    ring_len = 0 if ring is None else ring.numel() - 2
    if workspace is None:
        workspace = _workspace(x.device, hq_quantize_workspace_bytes(PER_TENSOR, rows, cols, True))
    check(lib.hq_quantize_fp8_transpose(_ptr(x), _DT[x.dtype], rows, cols, fmt, _ptr(qo), _ptr(qt), _ptr(scales),
                                        _ptr(amax_out), _ptr(multiplier), _ptr(ring), ring_len, ring_idx,
                                        ring_margin, _ptr(workspace), workspace.numel(), _stream(stream)))
    return qo, qt, scales


def hq_grad_bias_workspace_bytes(rows, cols):
    return lib.hq_grad_bias_workspace_bytes(rows, cols)


def hq_grad_bias(g, out=None, workspace=None, stream=None):
    """Bias gradient of a 2-D CUDA tensor g [rows, cols]: the column sums,
    accumulated in f32, in g's dtype ([cols]).  Returns out."""
    if g.dim() != 2:
        raise ValueError("g must be 2-D")
    if g.dtype not in _DT:
        raise ValueError("g must be float32, bfloat16 or float16")
    g = g.contiguous()
    rows, cols = g.shape
    if out is None:
        out = torch.empty((cols,), dtype=g.dtype, device=g.device)
    if workspace is None:
        workspace = _workspace(g.device, hq_grad_bias_workspace_bytes(rows, cols), slot="grad_bias")
    check(lib.hq_grad_bias(_ptr(g), _DT[g.dtype], rows, cols, _ptr(out), _ptr(workspace),
                           0 if workspace is None else workspace.numel(), _stream(stream)))
    return out


def hq_quantize_fp8_noalloc(x, fmt=E4M3, gran=PER_TOKEN, q=None, scales=None, amax_out=None, ring=None,
                            ring_idx=0, ring_margin=0, stream=None):
    """hq_quantize_fp8 for callers that cannot allocate device memory: the
    library's static scratch replaces the workspace (calls must not overlap
    on the GPU).  Returns (q, scales)."""
    if x.dim() != 2:
        raise ValueError("x must be 2-D")
    if x.dtype not in _DT:
        raise ValueError("x must be float32, bfloat16 or float16")
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")
    rows, cols = x.shape
    ns = hq_scale_count(gran, rows, cols)
    if q is None:
        q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((max(ns, 0),), dtype=torch.float32, device=x.device)
    ring_len = 0 if ring is None else ring.numel() - 2
    check(lib.hq_quantize_fp8_noalloc(_ptr(x), _DT[x.dtype], rows, cols, fmt, gran, _ptr(q), _ptr(scales),
                                      _ptr(amax_out), _ptr(ring), ring_len, ring_idx, ring_margin,
                                      _stream(stream)))
    return q, scales


def hq_gemm_a8w8(xq, wq, x_scale, w_scale, fmt=E4M3, out=None, stream=None):
    """out[M,N] bf16 = x_scale[m] * w_scale[n] * sum_k dec(xq[m,k]) dec(wq[n,k])."""
    xq, wq = xq.contiguous(), wq.contiguous()
    x_scale, w_scale = x_scale.contiguous(), w_scale.contiguous()
    M, K = xq.shape
    N = wq.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    check(lib.hq_gemm_a8w8(_ptr(xq), _ptr(wq), fmt, _ptr(x_scale), x_scale.numel(), _ptr(w_scale),
                           w_scale.numel(), M, N, K, _ptr(out), _stream(stream)))
    return out


def hq_gemm_a8w8_ex(xq, wq, x_scale, w_scale, fmt=E4M3, bias=None, out=None, q_out=None, q_fmt=E4M3,
                    q_scale=None, q_amax=None, ring=None, ring_idx=0, ring_margin=0, workspace=None, stream=None):
    """The a8w8 GEMM with the fused epilogues: an optional bf16 bias [N] added
    before the rounding, and either the bf16 out (default) or, with `ring`,
    FP8 codes of the bf16 result quantized per tensor with the delayed ring
    (bit-identical to hq_gemm_a8w8 + hq_quantize_fp8 with that ring).
    Returns out, or (q_out, q_scale) with a ring."""
    xq, wq = xq.contiguous(), wq.contiguous()
    x_scale, w_scale = x_scale.contiguous(), w_scale.contiguous()
    M, K = xq.shape
    N = wq.shape[0]
    ring_len = 0
    if ring is not None:
        ring_len = ring.numel() - 2
        if q_out is None:
            q_out = torch.empty((M, N), dtype=torch.uint8, device=xq.device)
        if q_scale is None:
            q_scale = torch.empty((1,), dtype=torch.float32, device=xq.device)
        if workspace is None:
            workspace = _workspace(xq.device, hq_quantize_workspace_bytes(PER_TENSOR, M, N, True))
    elif out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    check(lib.hq_gemm_a8w8_ex(_ptr(xq), _ptr(wq), fmt, _ptr(x_scale), x_scale.numel(), _ptr(w_scale),
                              w_scale.numel(), _ptr(bias), M, N, K, _ptr(out), _ptr(q_out), q_fmt, _ptr(q_scale),
                              _ptr(q_amax), _ptr(ring), ring_len, ring_idx, ring_margin, _ptr(workspace),
                              0 if workspace is None else workspace.numel(), _stream(stream)))
    return (q_out, q_scale) if ring is not None else out


def hq_gemm_a8w8_blockq(xq, wq, x_scale, w_scale, fmt=E4M3, bias=None, q_fmt=E4M3, block=32, q_out=None,
                        q_scales=None, stream=None):
    """The a8w8 GEMM (optional bf16 bias) with its bf16 result quantized
    block-wise in the epilogue: FP8 codes [M, N] and dequant scales
    [M, N / block] per 32-column block of a row (bit-identical to
    hq_gemm_a8w8_ex + hq_quantize_fp8_blockwise).  Returns (q_out, q_scales)."""
    xq, wq = xq.contiguous(), wq.contiguous()
    x_scale, w_scale = x_scale.contiguous(), w_scale.contiguous()
    M, K = xq.shape
    N = wq.shape[0]
    if q_out is None:
        q_out = torch.empty((M, N), dtype=torch.uint8, device=xq.device)
    if q_scales is None:
        q_scales = torch.empty((M, N // block if block > 0 else 0), dtype=torch.float32, device=xq.device)
    check(lib.hq_gemm_a8w8_blockq(_ptr(xq), _ptr(wq), fmt, _ptr(x_scale), x_scale.numel(), _ptr(w_scale),
                                  w_scale.numel(), _ptr(bias), M, N, K, _ptr(q_out), q_fmt, block, _ptr(q_scales),
                                  _stream(stream)))
    return q_out, q_scales


def hq_grouped_gemm_a8w8(xq, wq, x_scale, w_scale, offsets, fmt=E4M3, out=None, stream=None):
    """Per-expert a8w8 GEMM: rows [offsets[e], offsets[e+1]) of xq times wq[e]^T."""
    xq, wq = xq.contiguous(), wq.contiguous()
    x_scale, w_scale = x_scale.contiguous(), w_scale.contiguous()
    M, K = xq.shape
    E, N, _ = wq.shape
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    check(lib.hq_grouped_gemm_a8w8(_ptr(xq), _ptr(wq), fmt, _ptr(x_scale), x_scale.numel(), _ptr(w_scale),
                                   w_scale.numel(), _ptr(offsets), E, M, N, K, _ptr(out), _stream(stream)))
    return out


def hq_grouped_gemm_bf16(x, w, offsets, out=None, stream=None):
    """Per-expert bf16 GEMM with FP32 accumulation."""
    x, w = x.contiguous(), w.contiguous()
    M, K = x.shape
    E, N, _ = w.shape
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    check(lib.hq_grouped_gemm_bf16(_ptr(x), _ptr(w), _ptr(offsets), E, M, N, K, _ptr(out), _stream(stream)))
    return out


def hq_check_device_error():
    check(lib.hq_check_device_error())


def hq_version():
    return lib.hq_version().decode()
