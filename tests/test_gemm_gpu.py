"""GPU parity of the tcgen05 a8w8 GEMM against the oracle, through the C ABI,
plus the caller-owned-out contract of ROCm/aiter PR 6437 ("Technical
Details", "Test Plan"): a dense view into a larger buffer is written and the
rest is untouched; invalid outs raise and leave the buffer untouched; empty
out is a no-op; operands on the host are rejected; the output is
overwritten, never accumulated (megablocks-hip TODO-gg.md).

Tolerance (the pass criterion of the scaled GEMM): |out - ref| <=
8e-3 |ref| + 1e-3 max|ref| with ref the exact product rounded to bf16.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from fp8_dynamic_quantization_amax_b200 import _hq as H
from _gpu import assert_gemm_close, dev, dev_bf16, host, host_bits

pytestmark = pytest.mark.gpu


def rand_codes(rng, shape, fmt):
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    v = O.decode_array(c.reshape(-1), fmt)
    c.reshape(-1)[~np.isfinite(v)] = 0
    return c


def gemm_gpu(xq, wq, xs, ws, fmt):
    out = H.hq_gemm_a8w8(dev(xq), dev(wq), dev(xs), dev(ws), fmt)
    torch.cuda.synchronize()
    return host_bits(out)


SHAPES = [(1, 8, 16), (5, 8, 32), (128, 128, 128), (129, 136, 144), (200, 264, 512), (300, 256, 1040),
          (64, 1024, 256), (257, 2048, 384), (512, 4096, 256),
          # CTA-pair path (M >= 512, N % 256 == 0): M not a multiple of 256
          # (the second CTA's half partly or wholly past M), 9 N tiles, ragged K
          (600, 2304, 272), (700, 2048, 128), (1024, 2560, 512),
          # 256 x 512 CTA-pair tiles (M >= 8192, N % 512 == 0): a partial last M tile
          (8200, 2560, 32),
          # small-M (decode) paths: 64-wide tiles (16 / 64 A rows), 128-wide (64 A rows)
          (17, 2048, 384), (33, 520, 160), (24, 18944, 128)]

# Decode paths on a 148-SM B200, by tile width: 64 while N/64 tiles fit on
# the SMs, 128 while N/128 do, 208 up to 208 x 148 columns (a ragged last
# tile, a 16-column tail chunk per tile), 256 beyond; each with A loaded 16 /
# 64 / 128 rows per K block.
DECODE_SHAPES = [(120, 4096, 384),                                      # 64 / 128 rows
                 (10, 9600, 128), (90, 12000, 128),                     # 128 / 16 and 128 rows
                 (40, 19200, 256), (16, 19000, 256), (100, 19200, 128),  # 208 / 64, 16, 128 rows
                 (8, 30848, 64), (50, 30848, 64), (128, 30976, 64)]     # 256 / 16, 64, 128 rows


@pytest.mark.parametrize("fmt", [O.E4M3, O.E5M2])
@pytest.mark.parametrize("bcast", ["none", "x", "w", "both"])
def test_gemm_random_codes(fmt, bcast):
    for i, (M, N, K) in enumerate(SHAPES):
        rng = np.random.default_rng(100 + i)
        xq = rand_codes(rng, (M, K), fmt)
        wq = rand_codes(rng, (N, K), fmt)
        xs = rng.uniform(0.001, 0.01, 1 if bcast in ("x", "both") else M).astype(np.float32)
        ws = rng.uniform(0.001, 0.01, 1 if bcast in ("w", "both") else N).astype(np.float32)
        if fmt == O.E5M2:
            xs *= np.float32(1e-4)
            ws *= np.float32(1e-4)
        out = gemm_gpu(xq, wq, xs, ws, fmt)
        ref = O.gemm_a8w8(xq, wq, fmt, xs, ws)
        assert_gemm_close(out, ref)
    H.hq_check_device_error()


@pytest.mark.parametrize("fmt", [O.E4M3, O.E5M2])
def test_gemm_decode_tile_widths(fmt):
    for i, (M, N, K) in enumerate(DECODE_SHAPES):
        rng = np.random.default_rng(300 + i)
        xq = rand_codes(rng, (M, K), fmt)
        wq = rand_codes(rng, (N, K), fmt)
        xs = rng.uniform(0.001, 0.01, M).astype(np.float32)
        ws = rng.uniform(0.001, 0.01, N).astype(np.float32)
        if fmt == O.E5M2:
            xs *= np.float32(1e-4)
            ws *= np.float32(1e-4)
        out = gemm_gpu(xq, wq, xs, ws, fmt)
        assert_gemm_close(out, O.gemm_a8w8(xq, wq, fmt, xs, ws))
    H.hq_check_device_error()


def test_gemm_one_hot_selects_weight_columns():
    rng = np.random.default_rng(7)
    K, N = 256, 136
    wq = rand_codes(rng, (N, K), O.E4M3)
    xq = np.zeros((K, K), np.uint8)
    xq[np.arange(K), np.arange(K)] = 0x38  # 1.0
    xs = np.full(1, 0.5, np.float32)
    ws = rng.uniform(0.1, 1, N).astype(np.float32)
    out = gemm_gpu(xq, wq, xs, ws, O.E4M3)
    assert_gemm_close(out, O.gemm_a8w8(xq, wq, O.E4M3, xs, ws))


def test_gemm_k_zero_and_empty():
    xs = torch.ones(4, device="cuda")
    ws = torch.full((8,), -1.0, device="cuda")
    xq = torch.zeros((4, 16), dtype=torch.uint8, device="cuda")
    wq = torch.zeros((8, 16), dtype=torch.uint8, device="cuda")
    out = torch.full((4, 8), 3.0, dtype=torch.bfloat16, device="cuda")
    H.hq_gemm_a8w8(xq[:, :0], wq[:, :0], xs, ws, out=out)
    o = host_bits(out)
    assert (o == 0x8000).all()  # bf16(-0.0): 0 * (1 * -1)
    # M == 0 / N == 0: no-op on a valid buffer
    buf = torch.full((8,), 5.0, dtype=torch.bfloat16, device="cuda")
    H.check(H.lib.hq_gemm_a8w8(xq.data_ptr(), wq.data_ptr(), 0, xs.data_ptr(), 1, ws.data_ptr(), 8, 0, 8, 16,
                               buf.data_ptr(), None))
    H.check(H.lib.hq_gemm_a8w8(xq.data_ptr(), wq.data_ptr(), 0, xs.data_ptr(), 4, ws.data_ptr(), 1, 4, 0, 16,
                               buf.data_ptr(), None))
    torch.cuda.synchronize()
    assert (host(buf.float()) == 5.0).all()


def test_out_view_into_larger_buffer_and_rejections():
    rng = np.random.default_rng(9)
    M, N, K = 96, 136, 256
    xq, wq = rand_codes(rng, (M, K), O.E4M3), rand_codes(rng, (N, K), O.E4M3)
    xs = rng.uniform(0.01, 0.1, M).astype(np.float32)
    ws = rng.uniform(0.01, 0.1, N).astype(np.float32)
    ref = O.gemm_a8w8(xq, wq, O.E4M3, xs, ws)
    dxq, dwq, dxs, dws = dev(xq), dev(wq), dev(xs), dev(ws)
    canary = np.uint16(0xFFFF)
    buf = torch.full((M * N + 64,), -1, dtype=torch.int16, device="cuda")  # 0xFFFF everywhere
    off = 8  # 16 bytes
    view = buf[off:off + M * N].view(torch.bfloat16).view(M, N)
    H.hq_gemm_a8w8(dxq, dwq, dxs, dws, out=view)
    b = host(buf).view(np.uint16)
    assert (b[:off] == canary).all() and (b[off + M * N:] == canary).all()
    assert_gemm_close(b[off:off + M * N].reshape(M, N), ref)

    def raw(out_ptr, xq_ptr=dxq.data_ptr()):
        return H.lib.hq_gemm_a8w8(xq_ptr, dwq.data_ptr(), 0, dxs.data_ptr(), M, dws.data_ptr(), N, M, N, K,
                                  out_ptr, None)

    fresh = torch.full((M * N + 64,), -1, dtype=torch.int16, device="cuda")
    assert raw(fresh.data_ptr() + 2) == 2            # odd bf16 offset: MISALIGNED
    assert raw(dxq.data_ptr()) == 3                  # out over XQ: OVERLAP
    pinned = torch.empty(M * N, dtype=torch.int16).pin_memory()
    assert raw(pinned.data_ptr()) == 4               # host memory: WRONG_DEVICE
    host_x = torch.from_numpy(xq.copy())
    assert raw(fresh.data_ptr(), host_x.data_ptr()) == 4
    torch.cuda.synchronize()
    assert (host(fresh).view(np.uint16) == canary).all()


def test_overwrite_not_accumulate_and_strided_inputs():
    rng = np.random.default_rng(11)
    M, N, K = 130, 264, 384
    xq, wq = rand_codes(rng, (M, K), O.E4M3), rand_codes(rng, (N, K), O.E4M3)
    xs = rng.uniform(0.01, 0.1, M).astype(np.float32)
    ws = rng.uniform(0.01, 0.1, N).astype(np.float32)
    ref = O.gemm_a8w8(xq, wq, O.E4M3, xs, ws)
    out = torch.full((M, N), 1e30, dtype=torch.bfloat16, device="cuda")
    for _ in range(2):
        H.hq_gemm_a8w8(dev(xq), dev(wq), dev(xs), dev(ws), out=out)
        assert_gemm_close(host_bits(out), ref)
    # a column-major XQ (transposed storage) is made dense by the binding
    xq_t = dev(np.ascontiguousarray(xq.T)).t()
    assert not xq_t.is_contiguous()
    out2 = H.hq_gemm_a8w8(xq_t, dev(wq), dev(xs), dev(ws))
    np.testing.assert_array_equal(host_bits(out2), host_bits(out))


def test_tiny_pipeline_f32():
    # Tiny workload: X f32 [64,256] (rows 3 and 17 x50), W f32 [128,256];
    # per-token X, per-output-channel W (one scale per row of W[N,K]), E4M3.
    x, w = W.tiny()
    xq, xs = H.hq_quantize_fp8(dev(x), H.E4M3, H.PER_TOKEN)
    wq, ws = H.hq_quantize_fp8(dev(w), H.E4M3, H.PER_TOKEN)
    out = H.hq_gemm_a8w8(xq, wq, xs, ws, H.E4M3)
    torch.cuda.synchronize()
    xqo, xso, _ = O.quantize(x, O.E4M3, O.PER_TOKEN)
    wqo, wso, _ = O.quantize(w, O.E4M3, O.PER_TOKEN)
    np.testing.assert_array_equal(host(xq), xqo)
    np.testing.assert_array_equal(host(wq), wqo)
    np.testing.assert_array_equal(host(xs), xso)
    np.testing.assert_array_equal(host(ws), wso)
    assert_gemm_close(host_bits(out), O.gemm_a8w8(xqo, wqo, O.E4M3, xso, wso))


# ------------------------------------------------------------ large GEMM
@pytest.fixture(scope="module")
def large_w():
    """W bf16 [28672, 8192] ~N(0, 0.02), its device copy and the oracle's
    per-row (output-channel) quantization of all of it."""
    w = W.large_w(28672, 8192)
    wq_o, ws_o, _ = O.quantize(w, O.E4M3, O.PER_TOKEN)
    return w, wq_o, ws_o


@pytest.mark.parametrize("M", [1, 16, 128, 4096, 16384])
def test_large_gemm_pipeline(large_w, M):
    w, wq_o, ws_o = large_w
    N, K = w.shape
    x = W.large_x(M, K)
    xd, wd = dev_bf16(x), dev_bf16(w)
    xq, xs = H.hq_quantize_fp8(xd, H.E4M3, H.PER_TOKEN)
    wq, ws = H.hq_quantize_fp8(wd, H.E4M3, H.PER_TOKEN)
    del wd
    buf = torch.full((M * N + 64,), -1, dtype=torch.int16, device="cuda")
    out = buf[8:8 + M * N].view(torch.bfloat16).view(M, N)   # 16-byte offset in a caller buffer
    H.hq_gemm_a8w8(xq, wq, xs, ws, H.E4M3, out=out)
    torch.cuda.synchronize()
    H.hq_check_device_error()
    b = host(buf).view(np.uint16)
    assert (b[:8] == 0xFFFF).all() and (b[8 + M * N:] == 0xFFFF).all()
    # quantized weights: bit-exact on every row
    np.testing.assert_array_equal(host(ws), ws_o)
    rng = np.random.default_rng(M)
    wrows = rng.choice(N, 64, replace=False)
    np.testing.assert_array_equal(host(wq[torch.from_numpy(wrows).cuda()]), wq_o[wrows])
    # activations: oracle on sampled rows (per-token rows are independent)
    mrows = np.unique(np.concatenate([rng.choice(M, min(M, 48), replace=False), [0, M - 1]]))
    xqo, xso, _ = O.quantize(x[mrows], O.E4M3, O.PER_TOKEN)
    np.testing.assert_array_equal(host(xq[torch.from_numpy(mrows).cuda()]), xqo)
    np.testing.assert_array_equal(host(xs)[mrows], xso)
    o = b[8:8 + M * N].reshape(M, N)
    if M <= 16:
        ref = O.gemm_a8w8(xqo, wq_o, O.E4M3, xso, ws_o)          # every output
        assert_gemm_close(o[mrows], ref)
    else:
        ms = np.repeat(np.arange(mrows.size), 64)
        ns = rng.integers(0, N, ms.size)
        ref = O.gemm_a8w8_entries(xqo, wq_o, O.E4M3, xso, ws_o, ms, ns)
        # 2 full rows and 2 full columns as well
        full_rows = O.gemm_a8w8(xqo[:2], wq_o, O.E4M3, xso[:2], ws_o)
        cols = rng.choice(N, 2, replace=False)
        full_cols = O.gemm_a8w8(xqo, wq_o[cols], O.E4M3, xso, ws_o[cols])
        mx = max(np.abs(W.bf16_bits_to_f32(full_rows)).max(), np.abs(W.bf16_bits_to_f32(ref)).max())
        assert_gemm_close(o[mrows[ms], ns], ref, max_ref=mx)
        assert_gemm_close(o[mrows[:2]], full_rows, max_ref=mx)
        assert_gemm_close(o[mrows][:, cols], full_cols, max_ref=mx)


@pytest.mark.parametrize("M", [16, 4096])
def test_large_gemm_swapped_shape(M):
    # N = 8192, K = 28672 (the down projection of the same layer)
    N, K = 8192, 28672
    w = W.large_w(N, K, seed=2)
    x = W.large_x(M, K, seed=3)
    xq, xs = H.hq_quantize_fp8(dev_bf16(x), H.E4M3, H.PER_TOKEN)
    wq, ws = H.hq_quantize_fp8(dev_bf16(w), H.E4M3, H.PER_TOKEN)
    out = H.hq_gemm_a8w8(xq, wq, xs, ws, H.E4M3)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    mrows = rng.choice(M, min(M, 24), replace=False)
    nrows = rng.choice(N, 96, replace=False)
    xqo, xso, _ = O.quantize(x[mrows], O.E4M3, O.PER_TOKEN)
    wqo, wso, _ = O.quantize(w[nrows], O.E4M3, O.PER_TOKEN)
    np.testing.assert_array_equal(host(xq[torch.from_numpy(mrows).cuda()]), xqo)
    np.testing.assert_array_equal(host(wq[torch.from_numpy(nrows).cuda()]), wqo)
    ref = O.gemm_a8w8(xqo, wqo, O.E4M3, xso, wso)
    o = host_bits(out)[mrows][:, nrows]
    assert_gemm_close(o, ref)
    H.hq_check_device_error()
