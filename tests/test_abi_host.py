"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/hq.h declares, and rejects invalid arguments with a
status before any CUDA call (so fake pointer values are never touched).

Contract source: ROCm/aiter PR 6437 "Technical Details" (validation before
launch, 16-byte-aligned contiguous out, no overlap) and fuel-ir
quant_scale.rs (scale_count, as_str, ScalePair display strings).
"""
import ctypes
import os
import re
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

from fp8_dynamic_quantization_amax_b200 import _hq as H  # noqa: E402

L = H.lib
OK, INVALID, MISALIGNED, OVERLAP, TOO_LARGE = 0, 1, 2, 3, 8


def test_every_declared_symbol_is_exported():
    header = open(os.path.join(ROOT, "include", "hq.h")).read()
    declared = set(re.findall(r"\b(hq_[a-z0-9_]+)\s*\(", header))
    assert declared == set(H.EXPORTED)
    nm = subprocess.run(["nm", "-D", "--defined-only", H.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (hq_[a-z0-9_]+)\b", nm))
    assert declared <= exported, declared - exported
    for name in declared:
        assert hasattr(L, name)


def test_library_links_no_torch_and_no_driver_library():
    ldd = subprocess.run(["ldd", H.LIB_PATH], capture_output=True, text=True).stdout
    assert "libtorch" not in ldd and "libc10" not in ldd
    assert "libcuda.so" not in ldd  # driver reached through the runtime's entry-point query


def test_scale_count_and_names():
    # quant_scale.rs: scale_count(100, 200) = 1 / 100 / 200
    assert H.hq_scale_count(H.PER_TENSOR, 100, 200) == 1
    assert H.hq_scale_count(H.PER_TOKEN, 100, 200) == 100
    assert H.hq_scale_count(H.PER_CHANNEL, 100, 200) == 200
    assert H.hq_scale_count(7, 1, 1) == -1 and H.hq_scale_count(H.PER_TOKEN, -1, 2) == -1
    assert [H.hq_granularity_name(g) for g in (0, 1, 2)] == ["per_tensor", "per_token", "per_channel"]
    assert H.hq_granularity_name(3) is None
    assert H.hq_scale_pair_name(H.PER_TOKEN, H.PER_CHANNEL) == "act_per_token_weight_per_channel"
    assert H.hq_scale_pair_name(H.PER_TENSOR, H.PER_TENSOR) == "act_per_tensor_weight_per_tensor"
    buf = ctypes.create_string_buffer(8)
    assert L.hq_scale_pair_name(1, 2, buf, 8) == -1  # too short
    assert H.hq_version().startswith("hq ")


def test_workspace_sizes():
    assert H.hq_quantize_workspace_bytes(H.PER_TOKEN, 8192, 8192) == 0
    assert H.hq_quantize_workspace_bytes(H.PER_TENSOR, 8192, 8192) == 256
    assert H.hq_quantize_workspace_bytes(H.PER_TENSOR, 10, 10, delayed=True) == 256
    c = H.hq_quantize_workspace_bytes(H.PER_CHANNEL, 3, 8192)
    assert c >= 16 + 8 * 8192 and c % 256 == 0


# Fake device addresses: validation must reject before dereferencing.
BASE = 0x7F0000000000


def q(x=BASE, xt=H.BF16, rows=4, cols=64, fmt=H.E4M3, g=H.PER_TOKEN, qp=BASE + 0x100000,
      sc=BASE + 0x200000, am=None, ring=None, rl=0, ri=0, rm=0, ws=None, wsb=0):
    return L.hq_quantize_fp8(x, xt, rows, cols, fmt, g, qp, sc, am, ring, rl, ri, rm, ws, wsb, None)


def test_quantize_rejections():
    assert q(xt=5) == INVALID
    assert q(fmt=2) == INVALID
    assert q(g=3) == INVALID
    assert q(rows=-1) == INVALID
    assert q(rows=1 << 31) == TOO_LARGE
    assert q(rows=1 << 21, cols=1 << 20) == TOO_LARGE
    assert q(x=None) == INVALID
    assert q(qp=None) == INVALID
    assert q(sc=None) == INVALID
    # ring only with per-tensor; len >= 1; idx in range
    assert q(ring=BASE + 0x300000, rl=16, g=H.PER_TOKEN) == INVALID
    assert q(ring=BASE + 0x300000, rl=0, g=H.PER_TENSOR, ws=BASE + 0x400000, wsb=256) == INVALID
    assert q(ring=BASE + 0x300000, rl=16, ri=16, g=H.PER_TENSOR, ws=BASE + 0x400000, wsb=256) == INVALID
    assert q(ring=BASE + 0x300000, rl=16, ri=-1, g=H.PER_TENSOR, ws=BASE + 0x400000, wsb=256) == INVALID
    # workspace required and large enough
    assert q(g=H.PER_TENSOR) == INVALID
    assert q(g=H.PER_TENSOR, ws=BASE + 0x400000, wsb=16) == INVALID
    assert "workspace" in L.hq_last_error().decode()
    # alignment
    assert q(x=BASE + 1) == MISALIGNED
    assert q(xt=H.F32, x=BASE + 2) == MISALIGNED
    assert q(sc=BASE + 0x200002) == MISALIGNED
    assert q(g=H.PER_TENSOR, ws=BASE + 0x400010, wsb=512) == MISALIGNED
    # overlap: outputs with x, and with each other
    assert q(qp=BASE + 8) == OVERLAP
    assert q(sc=BASE + 0x100000 + 8) == OVERLAP
    assert q(am=BASE + 0x200000) == OVERLAP
    assert "overlaps" in L.hq_last_error().decode()
    # nothing to do: scale_count == 0 is accepted without touching anything
    assert q(rows=0, x=None, qp=None, sc=None) == OK


def g8(xq=BASE, wq=BASE + 0x1000000, fmt=H.E4M3, xs=BASE + 0x2000000, xsl=64, ws=BASE + 0x3000000, wsl=128,
       M=64, N=128, K=256, out=BASE + 0x4000000):
    return L.hq_gemm_a8w8(xq, wq, fmt, xs, xsl, ws, wsl, M, N, K, out, None)


def test_gemm_rejections():
    assert g8(fmt=9) == INVALID
    assert g8(M=-1) == INVALID
    assert g8(K=1 << 31) == TOO_LARGE
    assert g8(K=250) == INVALID          # rows must be whole 16-byte units
    assert g8(N=100) == INVALID          # 16-byte output rows
    assert g8(xsl=3) == INVALID and g8(wsl=64) == INVALID
    assert g8(xs=None) == INVALID and g8(out=None) == INVALID and g8(xq=None) == INVALID
    assert g8(out=BASE + 0x4000000 + 2) == MISALIGNED   # odd bf16 offset
    assert g8(out=BASE + 0x4000000 + 8) == MISALIGNED
    assert g8(xq=BASE + 8) == MISALIGNED
    assert g8(xs=BASE + 0x2000001) == MISALIGNED
    assert g8(out=BASE + 0x10) == OVERLAP                # out over XQ
    assert g8(out=BASE + 0x1000000) == OVERLAP           # out over WQ
    assert g8(out=BASE + 0x2000000 - 0x10) == OVERLAP    # out runs into x_scale


def gx(out=None, q_out=BASE + 0x4000000, q_fmt=H.E4M3, q_scale=BASE + 0x5000000, q_amax=None,
       ring=BASE + 0x5001000, ring_len=16, ring_idx=0, margin=0, ws=BASE + 0x5100000, wsb=256, bias=None,
       M=64, N=128, K=256):
    return L.hq_gemm_a8w8_ex(BASE, BASE + 0x1000000, H.E4M3, BASE + 0x2000000, 64, BASE + 0x3000000, 128, bias,
                             M, N, K, out, q_out, q_fmt, q_scale, q_amax, ring, ring_len, ring_idx, margin, ws, wsb,
                             None)


def test_fused_epilogue_rejections():
    # hq_gemm_a8w8_ex: exactly one output; the FP8 output follows the
    # delayed-quantize contract (ring, scale, zeroed workspace)
    assert gx(out=BASE + 0x6000000) == INVALID                 # both outputs
    assert gx(q_out=None) == INVALID                           # neither
    assert gx(ring=None) == INVALID and gx(q_scale=None) == INVALID and gx(ws=None) == INVALID
    assert gx(ring_idx=16) == INVALID and gx(ring_len=0) == INVALID and gx(margin=200) == INVALID
    assert gx(q_fmt=7) == INVALID and gx(wsb=64) == INVALID
    assert gx(N=24) == INVALID                                 # codes rows need N % 16 == 0
    assert gx(q_out=BASE + 0x4000008) == MISALIGNED
    assert gx(bias=BASE + 0x5200001) == MISALIGNED
    assert gx(ws=BASE + 0x5100010) == MISALIGNED
    assert gx(q_out=BASE + 0x10) == OVERLAP                    # codes over XQ
    assert gx(bias=BASE + 0x4000000) == OVERLAP                # codes over the bias
    assert gx(ring=BASE + 0x5000000) == OVERLAP                # ring over q_scale
    # the bf16 output with a bias keeps hq_gemm_a8w8's checks
    assert gx(out=BASE + 0x6000002, q_out=None, ring=None, ws=None, bias=BASE + 0x5200000) == MISALIGNED


def gbq(q_out=BASE + 0x4000000, q_fmt=H.E4M3, block=32, q_scales=BASE + 0x5000000, bias=None, M=64, N=128, K=256):
    return L.hq_gemm_a8w8_blockq(BASE, BASE + 0x1000000, H.E4M3, BASE + 0x2000000, 1, BASE + 0x3000000, 1, bias,
                                 M, N, K, q_out, q_fmt, block, q_scales, None)


def test_blockwise_output_rejections():
    # hq_gemm_a8w8_blockq: 32-column blocks only, whole blocks per row, codes
    # and scales caller-owned and apart from every input
    assert gbq(block=64) == INVALID and gbq(block=16) == INVALID and gbq(block=0) == INVALID
    assert gbq(N=112) == INVALID                               # 112 % 32 != 0
    assert gbq(q_out=None) == INVALID and gbq(q_scales=None) == INVALID
    assert gbq(q_fmt=3) == INVALID
    assert gbq(q_out=BASE + 0x4000008) == MISALIGNED
    assert gbq(q_scales=BASE + 0x5000002) == MISALIGNED
    assert gbq(bias=BASE + 0x5200001) == MISALIGNED
    assert gbq(q_out=BASE + 0x10) == OVERLAP                   # codes over XQ
    assert gbq(q_scales=BASE + 0x4000000 + 64 * 128 - 4) == OVERLAP   # scales run into the codes
    assert gbq(q_scales=BASE + 0x2000000) == OVERLAP           # scales over x_scale
    # the shape checks still apply to an empty result
    assert gbq(M=0, N=112, q_out=None, q_scales=None) == INVALID


def qtr(x=BASE, xt=H.BF16, rows=64, cols=128, fmt=H.E4M3, q=None, qt=BASE + 0x1000000, scales=BASE + 0x2000000,
        amax=None, mult=None, ring=None, ring_len=16, ring_idx=0, margin=0, ws=BASE + 0x3000000, wsb=256):
    return L.hq_quantize_fp8_transpose(x, xt, rows, cols, fmt, q, qt, scales, amax, mult, ring, ring_len, ring_idx,
                                       margin, ws, wsb, None)


def test_quantize_transpose_rejections():
    assert qtr(rows=72, cols=120) == INVALID          # both must be multiples of 16
    assert qtr(rows=60) == INVALID
    assert qtr(mult=BASE + 0x4000000, ring=BASE + 0x5000000) == INVALID   # one multiplier source
    assert qtr(ring=BASE + 0x5000000, ring_idx=16) == INVALID
    assert qtr(qt=None) == INVALID and qtr(scales=None) == INVALID and qtr(ws=None) == INVALID
    assert qtr(wsb=16) == INVALID and qtr(xt=7) == INVALID and qtr(fmt=5) == INVALID
    assert qtr(qt=BASE + 0x1000008) == MISALIGNED and qtr(x=BASE + 4) == MISALIGNED
    assert qtr(q=BASE + 0x4000004) == MISALIGNED and qtr(mult=BASE + 0x4000002) == MISALIGNED
    assert qtr(qt=BASE + 0x100) == OVERLAP            # transposed codes over x
    assert qtr(q=BASE + 0x1000000) == OVERLAP         # the two code buffers
    assert qtr(scales=BASE + 0x3000000 + 64) == OVERLAP  # scales inside the workspace


def test_stochastic_rejections():
    sr = L.hq_quantize_e5m2_stochastic

    def call(x=BASE, xt=H.BF16, rows=64, cols=128, g=H.PER_TENSOR, q=BASE + 0x1000000, s=BASE + 0x2000000,
             ws=BASE + 0x3000000, wsb=256):
        return sr(x, xt, rows, cols, g, 1234, q, s, None, ws, wsb, None)

    assert call(g=5) == INVALID and call(xt=9) == INVALID and call(rows=-1) == INVALID
    assert call(q=None) == INVALID and call(s=None) == INVALID and call(ws=None) == INVALID
    assert call(g=H.PER_CHANNEL, cols=100, wsb=1 << 16) == INVALID    # per-channel rows in 16-byte units
    assert call(x=BASE + 2) == MISALIGNED and call(q=BASE + 0x1000008) == MISALIGNED
    assert call(q=BASE + 0x40) == OVERLAP
    assert call(g=H.PER_TOKEN, ws=None, wsb=0, rows=0) == OK        # nothing to do (no scales)


def test_grouped_rejections():
    gg = L.hq_grouped_gemm_a8w8
    args = dict(xq=BASE, wq=BASE + 0x1000000, fmt=0, xs=BASE + 0x2000000, xsl=100, ws=BASE + 0x3000000,
                wsl=4 * 64, off=BASE + 0x5000000, E=4, M=100, N=64, K=128, out=BASE + 0x6000000)

    def call(**kw):
        a = dict(args, **kw)
        return gg(a["xq"], a["wq"], a["fmt"], a["xs"], a["xsl"], a["ws"], a["wsl"], a["off"], a["E"], a["M"],
                  a["N"], a["K"], a["out"], None)

    assert call(off=None) == INVALID
    assert call(E=0) == INVALID and call(E=2000) == INVALID
    assert call(wsl=64) == INVALID       # must be 1 or E*N
    assert call(off=BASE + 0x5000002) == MISALIGNED
    assert call(out=BASE + 0x5000000) == OVERLAP   # out over offsets
    b16 = L.hq_grouped_gemm_bf16
    assert b16(BASE, BASE + 0x1000000, None, 4, 100, 64, 128, BASE + 0x6000000, None) == INVALID
    assert b16(BASE, BASE + 0x1000000, BASE + 0x5000000, 4, 100, 64, 12, BASE + 0x6000000, None) == INVALID


def test_missing_library_fails_loudly(tmp_path):
    # A copy of the package without libhq.so must refuse to import: there is
    # no CPU or library fallback behind the binding.
    pkg = os.path.join(ROOT, "fp8_dynamic_quantization_amax_b200")
    dst = tmp_path / "fp8_dynamic_quantization_amax_b200"
    dst.mkdir()
    for f in ("__init__.py", "_hq.py"):
        shutil.copy(os.path.join(pkg, f), dst / f)
    r = subprocess.run([sys.executable, "-c", "import fp8_dynamic_quantization_amax_b200"], cwd=str(tmp_path),
                       capture_output=True, text=True)
    assert r.returncode != 0 and "libhq.so is not built" in r.stderr


def test_blockwise_rejections():
    bq = L.hq_quantize_fp8_blockwise

    def call(x=BASE, xt=H.BF16, rows=64, cols=128, fmt=H.E4M3, block=32, sr=0, q=BASE + 0x1000000,
             s=BASE + 0x2000000, a=None):
        return bq(x, xt, rows, cols, fmt, block, sr, 7, q, s, a, None)

    assert call(block=24) == INVALID and call(block=0) == INVALID and call(cols=120) == INVALID
    assert call(sr=1) == INVALID                      # stochastic rounding is E5M2-only
    assert call(xt=9) == INVALID and call(fmt=3) == INVALID and call(rows=-2) == INVALID
    assert call(q=None) == INVALID and call(s=None) == INVALID
    assert call(x=BASE + 2) == MISALIGNED and call(q=BASE + 0x1000008) == MISALIGNED
    assert call(s=BASE + 0x2000002) == MISALIGNED
    assert call(s=BASE + 0x100) == OVERLAP and call(a=BASE + 0x2000010) == OVERLAP
    assert call(rows=0, x=None, q=None, s=None) == OK
    dq = L.hq_dequantize_fp8_blockwise

    def dcall(q=BASE, fmt=H.E5M2, rows=64, cols=128, block=64, s=BASE + 0x1000000, ot=H.F32,
              out=BASE + 0x2000000):
        return dq(q, fmt, rows, cols, block, s, ot, out, None)

    assert dcall(ot=H.F16) == INVALID and dcall(block=8) == INVALID and dcall(cols=72) == INVALID
    assert dcall(out=None) == INVALID and dcall(s=None) == INVALID
    assert dcall(out=BASE + 0x2000004) == MISALIGNED and dcall(q=BASE + 8) == MISALIGNED
    assert dcall(out=BASE + 0x40) == OVERLAP and dcall(out=BASE + 0x1000000 - 0x100) == OVERLAP
    assert dcall(cols=0, q=None, s=None, out=None) == OK


def test_blockscaled_gemm_rejections():
    g = L.hq_gemm_blockscaled

    def call(xq=BASE, wq=BASE + 0x1000000, fmt=H.E4M3, xs=BASE + 0x2000000, ws=BASE + 0x3000000, block=32,
             bias=None, M=64, N=128, K=256, out=BASE + 0x4000000):
        return g(xq, wq, fmt, xs, ws, block, bias, M, N, K, out, None)

    assert call(block=16) == INVALID and call(block=48) == INVALID and call(block=0) == INVALID
    assert call(K=40) == INVALID and call(N=12) == INVALID and call(fmt=2) == INVALID and call(M=-1) == INVALID
    assert call(out=None) == INVALID and call(xs=None) == INVALID and call(wq=None) == INVALID
    assert call(out=BASE + 0x4000008) == MISALIGNED and call(xq=BASE + 4) == MISALIGNED
    assert call(bias=BASE + 0x5000004) == MISALIGNED and call(ws=BASE + 0x3000002) == MISALIGNED
    assert call(out=BASE + 0x100) == OVERLAP                 # out over A
    assert call(out=BASE + 0x2000000 - 0x100) == OVERLAP     # out running into x_scales
    assert call(bias=BASE + 0x4000000 + 0x40) == OVERLAP     # bias inside out
    assert call(M=1 << 31) == TOO_LARGE


def test_bounded_wait_probe_rejects_out_of_range_limits():
    assert L.hq_debug_bounded_wait(10, None) == INVALID             # below 1 us
    assert L.hq_debug_bounded_wait(3_000_000_000, None) == INVALID  # above 2 s


def test_delayed_batch_rejections():
    # argument checks of the batched delayed quantize, before any CUDA call
    L = H.lib

    def tensor(i, n=4096, ring_len=16, idx=0, margin=0, ring=True, ws=True, x=None):
        base = BASE + i * 0x10000000
        return H.DelayedTensor(base if x is None else x, n, base + 0x1000000, base + 0x2000000, None,
                               (base + 0x3000000) if ring else None, ring_len, idx, margin,
                               (base + 0x4000000) if ws else None, 256 if ws else 0)

    def call(ts, count=None, xt=H.BF16, fmt=H.E4M3):
        arr = (H.DelayedTensor * max(1, len(ts)))(*ts)
        return L.hq_quantize_fp8_delayed_batch(arr, len(ts) if count is None else count, xt, fmt, None)

    assert L.hq_quantize_fp8_delayed_batch(None, 1, H.BF16, H.E4M3, None) == INVALID
    assert call([tensor(0)], count=0) == INVALID and call([tensor(0)] * 9) == INVALID
    assert call([tensor(0)], xt=7) == INVALID and call([tensor(0)], fmt=5) == INVALID
    assert call([tensor(0), tensor(1, ring=False)]) == INVALID          # a delayed quantize needs a ring
    assert call([tensor(0, idx=16)]) == INVALID                         # ring_idx outside [0, len)
    assert call([tensor(0, margin=127)]) == INVALID
    assert call([tensor(0), tensor(1, ws=False)]) == INVALID            # no workspace
    assert call([tensor(0, x=BASE + 2 + 1)]) == MISALIGNED              # x not aligned to bf16
    t1 = tensor(1)
    t1.q = BASE + 0x1000000 + 64                                        # tensor 1's codes over tensor 0's
    assert call([tensor(0), t1]) == OVERLAP
    assert "tensor 1" in L.hq_last_error().decode()


def test_grad_bias_rejections():
    # argument checks of the bias gradient, before any CUDA call
    L = H.lib
    need = H.hq_grad_bias_workspace_bytes(100, 64)
    assert need == 256 + 4 * 64 * 4  # four bands (32 rows and more each) of partials, one strip counter (padded)
    assert H.hq_grad_bias_workspace_bytes(16384, 28672) == 256 * ((28672 // 256 * 4 + 255) // 256) + 64 * 28672 * 4
    assert H.hq_grad_bias_workspace_bytes(-1, 4) == 0
    g, out, ws = BASE, BASE + 0x1000000, BASE + 0x2000000
    assert L.hq_grad_bias(g, 9, 100, 64, out, ws, need, None) == INVALID            # dtype
    assert L.hq_grad_bias(g, H.BF16, -1, 64, out, ws, need, None) == INVALID        # shape
    assert L.hq_grad_bias(g, H.BF16, 1 << 31, 64, out, ws, need, None) == TOO_LARGE
    assert L.hq_grad_bias(g, H.BF16, 100, 64, None, ws, need, None) == INVALID      # no out
    assert L.hq_grad_bias(g, H.BF16, 100, 64, out, None, need, None) == INVALID     # no workspace
    assert L.hq_grad_bias(g, H.BF16, 100, 64, out, ws, need - 4, None) == INVALID   # workspace too small
    assert L.hq_grad_bias(g + 1, H.BF16, 100, 64, out, ws, need, None) == MISALIGNED
    assert L.hq_grad_bias(g, H.F32, 100, 64, out + 2, ws, need, None) == MISALIGNED
    assert L.hq_grad_bias(g, H.BF16, 100, 64, out, ws + 64, need, None) == MISALIGNED
    assert L.hq_grad_bias(g, H.BF16, 100, 64, g + 64, ws, need, None) == OVERLAP     # out inside g
    assert L.hq_grad_bias(g, H.BF16, 100, 64, out, g + 256, need, None) == OVERLAP   # workspace inside g
    assert L.hq_grad_bias(g, H.BF16, 100, 0, out, ws, need, None) == OK              # cols == 0: nothing to do
