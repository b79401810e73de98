"""GPU parity of the grouped (per-expert) GEMMs against the oracle, through the
C ABI: the a8w8 form (kind::f8f6f4) and the bf16 form with FP32
accumulation (kind::f16).  Expert row ranges come from device offsets;
empty experts, ragged counts that cross 128- and 256-row tiles (the 1-CTA
and the CTA-pair kernels), malformed offsets,
and the MoE workload (64 experts, K=2048, N=1408, 32768 tokens with Zipf(1.1)
counts and two empty experts) are covered.  Output is overwritten, never
accumulated (megablocks-hip TODO-gg.md).
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


CASES = [  # (counts per expert, N, K)
    ([3, 0, 130, 1, 0, 257], 64, 128),
    ([0, 0, 5], 8, 16),
    ([128, 128, 0, 64], 136, 272),
    ([300], 256, 384),
    ([40] * 20, 128, 256),
    # CTA-pair path (M_total >= 512, N >= 1024): 256-row tiles per expert,
    # experts of 300 / 257 / 520 rows (a partial second tile, 32-row groups
    # that straddle an expert boundary), a last N tile of 16 columns whose
    # second-CTA weight rows belong to the next expert, ragged K
    ([3, 0, 300, 1, 0, 257, 40], 1024, 256),
    ([520, 0, 17], 1040, 160),
    # N = 1408 with a ragged K and a partial 256-row tile in every expert
    ([520, 0, 17, 700], 1408, 96),
    # N = 1032: a last column tile of 8 columns (N % 16 = 8)
    ([300, 5, 260], 1032, 64),
]


@pytest.mark.parametrize("fmt", [O.E4M3, O.E5M2])
def test_grouped_a8w8_small(fmt):
    for i, (counts, N, K) in enumerate(CASES):
        rng = np.random.default_rng(40 + i)
        E = len(counts)
        off = np.zeros(E + 1, np.int32)
        off[1:] = np.cumsum(counts)
        M = int(off[-1])
        xq = rand_codes(rng, (M, K), fmt)
        wq = rand_codes(rng, (E, N, K), fmt)
        xs = rng.uniform(0.001, 0.01, M).astype(np.float32)
        ws = rng.uniform(0.001, 0.01, (E, N)).astype(np.float32)
        if fmt == O.E5M2:
            xs *= np.float32(1e-4)
        buf = torch.full((M * N + 16,), -1, dtype=torch.int16, device="cuda")
        out = buf[:M * N].view(torch.bfloat16).view(M, N)
        for _ in range(2):  # second call overwrites with the same values
            H.hq_grouped_gemm_a8w8(dev(xq), dev(wq), dev(xs), dev(ws), dev(off), fmt, out=out)
            torch.cuda.synchronize()
            ref = O.grouped_gemm_a8w8(xq, wq, fmt, xs, ws, off)
            if M:
                assert_gemm_close(host_bits(out), ref)
        assert (host(buf)[M * N:].view(np.uint16) == 0xFFFF).all()
    H.hq_check_device_error()


def test_grouped_bf16_small():
    for i, (counts, N, K) in enumerate(CASES):
        rng = np.random.default_rng(60 + i)
        E = len(counts)
        off = np.zeros(E + 1, np.int32)
        off[1:] = np.cumsum(counts)
        M = int(off[-1])
        x = W.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
        w = W.f32_to_bf16_bits(rng.standard_normal((E, N, K)).astype(np.float32) * np.float32(0.05))
        out = H.hq_grouped_gemm_bf16(dev_bf16(x), dev_bf16(w), dev(off))
        torch.cuda.synchronize()
        if M:
            assert_gemm_close(host_bits(out), O.grouped_gemm_bf16(x, w, off))
    H.hq_check_device_error()


def test_malformed_offsets_flagged_without_stray_writes():
    rng = np.random.default_rng(3)
    M, N, K, E = 64, 64, 128, 3
    xq, wq = rand_codes(rng, (M, K), O.E4M3), rand_codes(rng, (E, N, K), O.E4M3)
    xs, ws = np.ones(M, np.float32), np.ones(E * N, np.float32)
    buf = torch.full((M * N + 4096,), -1, dtype=torch.int16, device="cuda")
    out = buf[:M * N].view(torch.bfloat16).view(M, N)
    bad = np.array([0, 50, 10, 1000], np.int32)  # decreasing and beyond M
    H.hq_grouped_gemm_a8w8(dev(xq), dev(wq), dev(xs), dev(ws), dev(bad), O.E4M3, out=out)
    with pytest.raises(H.HQError) as ei:
        H.hq_check_device_error()
    assert ei.value.status == 1
    assert (host(buf)[M * N:].view(np.uint16) == 0xFFFF).all()
    H.hq_check_device_error()  # the word was cleared


@pytest.fixture(scope="module")
def moe():
    x, w, off = W.moe_inputs()
    return x, w, off


def _sample_rows(off, rng, per_expert=3):
    rows = []
    for e in range(off.size - 1):
        a, b = int(off[e]), int(off[e + 1])
        if b > a:
            rows += sorted(set([a, b - 1] + list(rng.integers(a, b, per_expert))))
    return np.array(rows, np.int64)


def test_moe_a8w8_full_size(moe):
    x, w, off = moe
    E, N, K = w.shape
    xq, xs = H.hq_quantize_fp8(dev_bf16(x), H.E4M3, H.PER_TOKEN)
    wq, ws = H.hq_quantize_fp8(dev_bf16(w.reshape(E * N, K)), H.E4M3, H.PER_TOKEN)
    out = H.hq_grouped_gemm_a8w8(xq, wq.view(E, N, K), xs, ws, dev(off), H.E4M3)
    torch.cuda.synchronize()
    H.hq_check_device_error()
    rng = np.random.default_rng(1)
    rows = _sample_rows(off, rng)
    xqo, xso, _ = O.quantize(x[rows], O.E4M3, O.PER_TOKEN)
    np.testing.assert_array_equal(host(xq[torch.from_numpy(rows).cuda()]), xqo)
    np.testing.assert_array_equal(host(xs)[rows], xso)
    o = host_bits(out)
    experts = np.searchsorted(off, rows, side="right") - 1
    refs, gots = [], []
    for e in np.unique(experts):
        sel = np.nonzero(experts == e)[0]
        nsel = rng.choice(N, 64, replace=False)
        wqo, wso, _ = O.quantize(w[e][nsel], O.E4M3, O.PER_TOKEN)
        np.testing.assert_array_equal(host(ws)[e * N + nsel], wso)
        refs.append(O.gemm_a8w8(xqo[sel], wqo, O.E4M3, xso[sel], wso).reshape(-1))
        gots.append(o[rows[sel]][:, nsel].reshape(-1))
    assert_gemm_close(np.concatenate(gots), np.concatenate(refs))


def test_moe_bf16_full_size(moe):
    x, w, off = moe
    E, N, K = w.shape
    out = H.hq_grouped_gemm_bf16(dev_bf16(x), dev_bf16(w), dev(off))
    torch.cuda.synchronize()
    H.hq_check_device_error()
    rng = np.random.default_rng(2)
    rows = _sample_rows(off, rng, per_expert=2)
    experts = np.searchsorted(off, rows, side="right") - 1
    # a mini grouped problem holding only the sampled rows, same experts
    counts = np.bincount(experts, minlength=E)
    moff = np.zeros(E + 1, np.int32)
    moff[1:] = np.cumsum(counts)
    nsel = rng.choice(N, 128, replace=False)
    ref = O.grouped_gemm_bf16(x[rows], np.ascontiguousarray(w[:, nsel, :]), moff)
    assert_gemm_close(host_bits(out)[rows][:, nsel], ref)
