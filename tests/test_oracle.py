"""Pins for the CPU oracle: each test checks it against something other than
itself -- the format facts the pages print, hand-computed traces, closed
forms, an independent library (ml_dtypes, torch) on the range where that
library's semantics coincide, or exact brute force (Python integers,
fractions) on tiny inputs.

Sources: hip-quant 0.6.0 README ("FP8 Formats", "Training-path numerical
guards"), fuel-ir quant_scale.rs (ScaleGranularity::scale_count and its
unit test), AstrAI ops.cu (ring commit message, mm_fp8), ROCm/aiter PR 6437
(Technical Details), megablocks-hip TODO-gg.md (overwrite, not accumulate).
"""
import math
import os
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
FMTS = [O.E4M3, O.E5M2]
ML = {O.E4M3: ml_dtypes.float8_e4m3fn, O.E5M2: ml_dtypes.float8_e5m2}


# ------------------------------------------------------------ format facts
def test_known_codes_golden():
    n = 0
    for line in open(os.path.join(GOLDEN, "fp8_known_codes.txt")):
        if line.startswith("#") or not line.strip():
            continue
        f, v, c = line.split()
        fmt = O.E4M3 if f == "E4M3" else O.E5M2
        code = int(c, 16)
        assert O.encode_sat(float(v), fmt) == code, line
        dv = O.decode(code, fmt)
        assert dv == float(v) and math.copysign(1, dv) == math.copysign(1, float(v)), line
        n += 1
    assert n >= 20


def test_format_limits():
    # hip-quant README "FP8 Formats": E4M3 max 448 and NaN only; E5M2 max
    # 57344 with +-Inf and NaN.
    assert O.fmax(O.E4M3) == 448.0 and O.fmax(O.E5M2) == 57344.0
    e4 = O.decode_array(np.arange(256, dtype=np.uint8), O.E4M3)
    e5 = O.decode_array(np.arange(256, dtype=np.uint8), O.E5M2)
    assert np.isnan(e4).sum() == 2 and np.isnan(e4[[0x7F, 0xFF]]).all()
    assert not np.isinf(e4).any()
    assert np.nanmax(e4) == 448.0 and np.nanmin(e4) == -448.0
    assert np.isinf(e5).sum() == 2 and e5[0x7C] == np.inf and e5[0xFC] == -np.inf
    assert np.isnan(e5).sum() == 6
    fin5 = e5[np.isfinite(e5)]
    assert fin5.max() == 57344.0 and fin5.min() == -57344.0
    # bias: 1.0 has exponent field == bias
    assert (0x38 >> 3) == 7 and (0x3C >> 2) == 15


@pytest.mark.parametrize("fmt", FMTS)
def test_decode_matches_ml_dtypes(fmt):
    codes = np.arange(256, dtype=np.uint8)
    ours = O.decode_array(codes, fmt)
    theirs = codes.view(ML[fmt]).astype(np.float64)
    both_nan = np.isnan(ours) & np.isnan(theirs)
    assert (both_nan | (ours == theirs)).all()
    assert (np.signbit(ours) == np.signbit(theirs))[~both_nan].all()


@pytest.mark.parametrize("fmt", FMTS)
def test_round_trip_all_codes(fmt):
    fmax = O.fmax(fmt)
    for c in range(256):
        v = O.decode(c, fmt)
        if math.isnan(v):
            assert O.encode_sat(v, fmt) == 0x7F  # canonical NaN (reading)
        elif math.isinf(v):
            # saturating cast: +-Inf -> +-max code
            assert O.encode_sat(v, fmt) == (0x80 if v < 0 else 0) | O.encode_sat(fmax, fmt)
        else:
            assert O.encode_sat(v, fmt) == c, hex(c)


@pytest.mark.parametrize("fmt", FMTS)
def test_codes_monotone(fmt):
    pos = [O.decode(c, fmt) for c in range(0x80)]
    pos = [v for v in pos if math.isfinite(v)]
    assert all(a < b for a, b in zip(pos, pos[1:]))


def _structured_f32():
    """Every (sign, exponent, top-7-mantissa) pattern with several low-16-bit
    tails: covers every rounding position (round bit plus sticky) of both
    formats, normals and subnormals, ties and near-ties."""
    hi = np.arange(1 << 16, dtype=np.uint32) << 16
    rng = np.random.default_rng(123)
    tails = [0x0000, 0x0001, 0x7FFF, 0x8000, 0x8001, 0xFFFF] + list(
        rng.integers(0, 1 << 16, size=4))
    u = (hi[:, None] | np.array(tails, np.uint32)[None, :]).reshape(-1)
    return u.view(np.float32)


@pytest.mark.parametrize("fmt", FMTS)
def test_encode_vs_ml_dtypes_in_range(fmt):
    # ml_dtypes casts are round-to-nearest-even but do not saturate, so they
    # pin the oracle wherever |y| < fmax.
    y = _structured_f32()
    fmax = O.fmax(fmt)
    ours = O.encode_sat_array(y, fmt)
    with np.errstate(all="ignore"):
        inr = np.isfinite(y) & (np.abs(y.astype(np.float64)) < fmax)
        theirs = y[inr].astype(ML[fmt]).view(np.uint8)
    assert inr.sum() > 100000
    bad = np.nonzero(ours[inr] != theirs)[0]
    assert bad.size == 0, (y[inr][bad[:5]], ours[inr][bad[:5]], theirs[bad[:5]])


@pytest.mark.parametrize("fmt", FMTS)
def test_encode_saturates_and_nan(fmt):
    y = _structured_f32()
    fmax = O.fmax(fmt)
    ours = O.encode_sat_array(y, fmt)
    maxc = O.encode_sat(fmax, fmt)
    with np.errstate(all="ignore"):
        big = ~np.isnan(y) & (np.abs(y.astype(np.float64)) >= fmax)
    expect = np.where(np.signbit(y[big]), 0x80 | maxc, maxc).astype(np.uint8)
    assert (ours[big] == expect).all()
    assert (ours[np.isnan(y)] == 0x7F).all()
    # just above fmax by one f32 ulp, and infinities
    up = np.nextafter(np.float32(fmax), np.float32(np.inf))
    assert O.encode_sat(float(up), fmt) == maxc
    assert O.encode_sat(float("inf"), fmt) == maxc
    assert O.encode_sat(float("-inf"), fmt) == 0x80 | maxc


# ------------------------------------------------------------- scale_count
def test_scale_count_quant_scale_rs():
    # fuel-ir quant_scale.rs, test scale_count_matches_granularity
    assert O.scale_count(O.PER_TENSOR, 100, 200) == 1
    assert O.scale_count(O.PER_TOKEN, 100, 200) == 100
    assert O.scale_count(O.PER_CHANNEL, 100, 200) == 200


# --------------------------------------------------------- amax and scale
def _bf16(a):
    return W.f32_to_bf16_bits(np.asarray(a, np.float32))


@pytest.mark.parametrize("fmt", FMTS)
def test_constant_row_closed_form(fmt):
    # A row of 3.5: amax 3.5, m = fmax/3.5 is a power of two times... exact:
    # 448/3.5 = 128, 57344/3.5 = 16384.  Every code is the max code.
    x = np.full((3, 16), 3.5, np.float32)
    x[1] = -3.5
    q, s, am = O.quantize(x, fmt, O.PER_TOKEN)
    m = O.fmax(fmt) / 3.5
    assert m == int(m)
    assert (am == 3.5).all()
    np.testing.assert_array_equal(s, np.float32(1.0 / m))
    maxc = O.encode_sat(O.fmax(fmt), fmt)
    assert (q[0] == maxc).all() and (q[1] == (0x80 | maxc)).all()


@pytest.mark.parametrize("fmt", FMTS)
def test_zero_row_and_signed_zero(fmt):
    x = np.zeros((2, 8), np.float32)
    x[1, 3] = -0.0
    x[1, 5] = 2.0
    q, s, am = O.quantize(x, fmt, O.PER_TOKEN)
    assert (q[0] == 0).all() and s[0] == 1.0 and am[0] == 0.0
    assert q[1, 3] == 0x80 and q[1, 0] == 0
    assert q[1, 5] == O.encode_sat(O.fmax(fmt), fmt)


@pytest.mark.parametrize("fmt", FMTS)
def test_power_of_two_scales(fmt):
    # amax = 2^k gives m = fmax * 2^-k exactly; values 2^j map to exact codes.
    x = np.array([[2.0 ** j for j in range(-3, 5)]], np.float32)
    q, s, am = O.quantize(x, fmt, O.PER_TENSOR)
    m = O.fmax(fmt) / 16.0
    assert am[0] == 16.0 and s[0] == np.float32(1.0 / m)
    for j, c in zip(range(-3, 5), q[0]):
        assert O.decode(int(c), fmt) == 2.0 ** j * m


@pytest.mark.parametrize("fmt", FMTS)
def test_nonfinite_skipped_by_amax(fmt):
    # hip-quant README "Training-path numerical guards": non-finite amax
    # samples are ignored.  Inf still saturates, NaN stays NaN.
    x = np.array([[1.0, np.nan, np.inf, -np.inf, 0.25]], np.float32)
    q, s, am = O.quantize(x, fmt, O.PER_TOKEN)
    maxc = O.encode_sat(O.fmax(fmt), fmt)
    assert am[0] == 1.0
    assert list(q[0]) == [maxc, 0x7F, maxc, 0x80 | maxc, O.encode_sat(O.fmax(fmt) / 4, fmt)]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("gran", [O.PER_TENSOR, O.PER_TOKEN, O.PER_CHANNEL])
def test_amax_element_hits_max_code(fmt, gran):
    # x = amax gives fmax (rounded), which encodes to the max code.
    rng = np.random.default_rng(5)
    x = _bf16(rng.standard_normal((17, 40)).astype(np.float32))
    q, s, am = O.quantize(x, fmt, gran)
    xf = W.bf16_bits_to_f32(x)
    maxc = O.encode_sat(O.fmax(fmt), fmt)
    ax = np.abs(xf)
    if gran == O.PER_TENSOR:
        r, c = np.unravel_index(np.argmax(ax), ax.shape)
        assert q[r, c] & 0x7F == maxc
        assert am[0] == ax.max()
    elif gran == O.PER_TOKEN:
        for r in range(17):
            c = np.argmax(ax[r])
            assert q[r, c] & 0x7F == maxc and am[r] == ax[r].max()
    else:
        for c in range(40):
            r = np.argmax(ax[:, c])
            assert q[r, c] & 0x7F == maxc and am[c] == ax[:, c].max()


@pytest.mark.parametrize("gran", [O.PER_TENSOR, O.PER_TOKEN, O.PER_CHANNEL])
def test_quantize_vs_torch_f32_pipeline(gran):
    # Independent restatement on the in-range part: amax by numpy, m by f32
    # division, y by f32 multiply, code by ml_dtypes (never saturates here
    # because |y| <= fmax up to f32 rounding, which the encode handles).
    rng = np.random.default_rng(7)
    xf = rng.standard_normal((33, 65)).astype(np.float32) * np.float32(3.0)
    for fmt in FMTS:
        q, s, am = O.quantize(xf, fmt, gran)
        axis = {O.PER_TENSOR: None, O.PER_TOKEN: 1, O.PER_CHANNEL: 0}[gran]
        a = np.abs(xf).max(axis=axis, keepdims=True).astype(np.float32)
        m = (np.float32(O.fmax(fmt)) / a).astype(np.float32)
        y = (xf * m).astype(np.float32)
        y = np.clip(y, -O.fmax(fmt), O.fmax(fmt)).astype(np.float32)
        ref = y.astype(ML[fmt]).view(np.uint8)
        np.testing.assert_array_equal(q, ref)
        np.testing.assert_array_equal(s, (np.float32(1) / m).reshape(-1))


def test_multiplier_degenerate():
    assert O.multiplier(0.0, O.E4M3) == 1.0
    # a subnormal amax makes fmax/amax overflow f32 -> m = 1 (reading)
    assert O.multiplier(1e-45, O.E4M3) == 1.0
    assert O.multiplier(1e-45, O.E5M2) == 1.0
    assert O.multiplier(448.0, O.E4M3) == 1.0
    assert O.multiplier(1.0, O.E5M2) == 57344.0


def test_bad_ring_args_rejected():
    x = np.ones((2, 4), np.float32)
    ring = np.array([0, 0, 1, 0], np.float32)
    with pytest.raises(ValueError):
        O.quantize(x, O.E4M3, O.PER_TOKEN, ring=ring)
    with pytest.raises(ValueError):
        O.quantize(x, O.E4M3, O.PER_TENSOR, ring=ring, ring_idx=2)


# -------------------------------------------------------------------- ring
def _parse_ring_golden():
    steps = []
    for line in open(os.path.join(GOLDEN, "ring_trace.txt")):
        if not line.startswith("step"):
            continue
        head, xs, codes, scale, ring = [p.strip() for p in line.split("|")]
        h = head.split()
        num, den = scale.split("/")
        steps.append(dict(idx=int(h[3]), margin=int(h[5]),
                          x=np.array([float(v) for v in xs.split()], np.float32),
                          codes=[int(c, 16) for c in codes.split()],
                          scale=np.float32(np.float32(num) / np.float32(den)),
                          ring=np.array([float(v) for v in ring.split()], np.float32)))
    return steps


def test_ring_hand_trace():
    ring = np.array([0, 0, 1, 0], np.float32)
    steps = _parse_ring_golden()
    assert len(steps) == 11
    for st in steps:
        x = st["x"].copy()
        q, s, am = O.quantize(x.reshape(1, 4), O.E4M3, O.PER_TENSOR, ring=ring,
                              ring_idx=st["idx"], ring_margin=st["margin"])
        assert list(q[0]) == st["codes"], (st, q)
        assert s[0] == st["scale"]
        np.testing.assert_array_equal(ring, st["ring"])


def test_ring_resume_bit_identical():
    # Checkpoint/resume: the ring is the only state; saving its len+2 floats
    # and restoring them gives a bit-identical continuation.
    L = 16
    rng = np.random.default_rng(11)
    xs = [W.f32_to_bf16_bits(rng.standard_normal((4, 32)).astype(np.float32)
                             * np.float32(0.5 * 16 ** (t / 39))) for t in range(40)]
    ring_a = np.zeros(L + 2, np.float32)
    ring_a[L] = 1.0
    outs_a = []
    for t, x in enumerate(xs):
        outs_a.append(O.quantize(x, O.E4M3, O.PER_TENSOR, ring=ring_a, ring_idx=t % L)[0])
    ring_b = np.zeros(L + 2, np.float32)
    ring_b[L] = 1.0
    for t in range(20):
        O.quantize(xs[t], O.E4M3, O.PER_TENSOR, ring=ring_b, ring_idx=t % L)
    saved = ring_b.tobytes()
    ring_c = np.frombuffer(saved, np.float32).copy()
    for t in range(20, 40):
        q = O.quantize(xs[t], O.E4M3, O.PER_TENSOR, ring=ring_c, ring_idx=t % L)[0]
        np.testing.assert_array_equal(q, outs_a[t])
    np.testing.assert_array_equal(ring_c, ring_a)


# -------------------------------------------------------------------- bf16
def test_double_to_bf16_vs_torch_on_f32_values():
    # For values exactly representable in f32, torch's f32 -> bf16 cast is a
    # single round-to-nearest-even: an independent pin.
    u = _structured_f32().view(np.uint32)
    u = u[(u & 0x7F800000) != 0x7F800000]  # finite only
    y = u.view(np.float32)[::7]
    ours = np.array([O.double_to_bf16(float(v)) for v in y], np.uint16)
    theirs = torch.from_numpy(y.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, theirs)


def test_double_to_bf16_single_rounding():
    # 1 + 2^-8 + 2^-40 is above the midpoint of [1, 1+2^-7]: rounds up.  A
    # double-rounding path through f32 (which keeps 1+2^-8, a tie) would give
    # 1.0 instead.
    assert O.double_to_bf16(1.0 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81
    assert O.double_to_bf16(1.0 + 2.0 ** -8) == 0x3F80          # tie -> even
    assert O.double_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82      # tie -> even
    assert O.double_to_bf16(-(1.0 + 2.0 ** -8 + 2.0 ** -40)) == 0xBF81
    assert O.double_to_bf16(3.4e38) == 0x7F80                   # overflow -> Inf
    assert O.double_to_bf16(2.0 ** -133) == 0x0001              # bf16 subnormal
    assert O.double_to_bf16(0.0) == 0 and O.double_to_bf16(-0.0) == 0x8000


# -------------------------------------------------------------------- GEMM
def _rand_codes(rng, shape, fmt):
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    bad = np.isnan(O.decode_array(c, fmt)) | np.isinf(O.decode_array(c, fmt))
    c.reshape(-1)[bad.reshape(-1)] = 0
    return c


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("MNK", [(1, 1, 1), (1, 1, 32), (3, 5, 7), (8, 16, 64), (5, 3, 300)])
def test_gemm_vs_exact_python_integers(fmt, MNK):
    # Brute force with exact Python integers: value(code) = n * 2^-f.
    M, N, K = MNK
    rng = np.random.default_rng(M * 100 + N * 10 + K + fmt)
    xq = _rand_codes(rng, (M, K), fmt)
    wq = _rand_codes(rng, (N, K), fmt)
    xs = rng.uniform(0.01, 2, M).astype(np.float32)
    ws = rng.uniform(0.01, 2, N).astype(np.float32)
    out, ref = O.gemm_a8w8(xq, wq, fmt, xs, ws, return_ref=True)
    frac = 9 if fmt == O.E4M3 else 16
    dx = xq.view(ML[fmt]).astype(np.float64)
    dw = wq.view(ML[fmt]).astype(np.float64)
    ix = [[int(v * 2 ** frac) for v in row] for row in dx]
    iw = [[int(v * 2 ** frac) for v in row] for row in dw]
    for m in range(M):
        for n in range(N):
            s = sum(a * b for a, b in zip(ix[m], iw[n]))
            exact = Fraction(s, 2 ** (2 * frac)) * Fraction(float(xs[m])) * Fraction(float(ws[n]))
            assert abs(Fraction(ref[m, n]) - exact) <= abs(exact) * Fraction(1, 2 ** 50)
            # bf16 of the exact value: nearest of the bf16 neighbours
            assert out[m, n] == _nearest_bf16(exact)


def _nearest_bf16(v: Fraction) -> int:
    f = float(v)
    b = int(torch.tensor([f], dtype=torch.float32).to(torch.bfloat16).view(torch.int16).item()) & 0xFFFF
    cands = {(b + d) & 0xFFFF for d in (-2, -1, 0, 1, 2)}
    best = None
    for c in cands:
        cv = np.array([c], np.uint16)
        val = float(W.bf16_bits_to_f32(cv)[0])
        if not math.isfinite(val):
            continue
        d = abs(Fraction(val) - v)
        key = (d, c & 1)  # ties -> even mantissa
        if best is None or key < best[0]:
            best = (key, c)
    return best[1]


@pytest.mark.parametrize("fmt", FMTS)
def test_gemm_vs_numpy_double(fmt):
    # E4M3 and E5M2 products and sums of K=64 terms are exact in fp64, so a
    # plain float64 matmul of ml_dtypes-decoded operands must agree exactly.
    rng = np.random.default_rng(3)
    M, N, K = 16, 24, 64
    xq = _rand_codes(rng, (M, K), fmt)
    wq = _rand_codes(rng, (N, K), fmt)
    if fmt == O.E5M2:  # keep the sum inside 53 bits
        xq &= 0xBF
        wq &= 0xBF
    xs = rng.uniform(0.5, 2, M).astype(np.float32)
    ws = rng.uniform(0.5, 2, N).astype(np.float32)
    _, ref = O.gemm_a8w8(xq, wq, fmt, xs, ws, return_ref=True)
    S = xq.view(ML[fmt]).astype(np.float64) @ wq.view(ML[fmt]).astype(np.float64).T
    expect = xs.astype(np.float64)[:, None] * ws.astype(np.float64)[None, :] * S
    np.testing.assert_array_equal(ref, expect)


def test_gemm_identity_like_and_broadcast_scales():
    # One-hot XQ rows with code 0x38 (= 1.0) select a column of WQ: out[m,n]
    # = bf16(xs * ws[n] * dec(WQ[n, k_m])).  Scales of length 1 broadcast.
    rng = np.random.default_rng(9)
    K, N = 32, 8
    wq = _rand_codes(rng, (N, K), O.E4M3)
    xq = np.zeros((K, K), np.uint8)
    xq[np.arange(K), np.arange(K)] = 0x38
    ws = rng.uniform(0.1, 1, N).astype(np.float32)
    out = O.gemm_a8w8(xq, wq, O.E4M3, np.array([2.0], np.float32), ws)
    for m in range(K):
        for n in range(N):
            v = 2.0 * float(ws[n]) * O.decode(int(wq[n, m]), O.E4M3)
            assert out[m, n] == O.double_to_bf16(v)


@pytest.mark.parametrize("fmt", FMTS)
def test_gemm_bias_vs_exact_fractions(fmt):
    # out = bf16 of the exact x_scale * w_scale * S + bias (bias a bf16 vector,
    # added before the single rounding), against exact rationals.
    rng = np.random.default_rng(31 + fmt)
    M, N, K = 4, 6, 40
    xq = _rand_codes(rng, (M, K), fmt)
    wq = _rand_codes(rng, (N, K), fmt)
    xs = rng.uniform(0.01, 2, M).astype(np.float32)
    ws = rng.uniform(0.01, 2, N).astype(np.float32)
    bias = W.f32_to_bf16_bits(rng.standard_normal(N).astype(np.float32) * np.float32(3.0))
    out = O.gemm_a8w8_bias(xq, wq, fmt, xs, ws, bias)
    frac = 9 if fmt == O.E4M3 else 16
    dx = xq.view(ML[fmt]).astype(np.float64)
    dw = wq.view(ML[fmt]).astype(np.float64)
    bv = W.bf16_bits_to_f32(bias)
    for m in range(M):
        for n in range(N):
            s = sum(int(a * 2 ** frac) * int(b * 2 ** frac) for a, b in zip(dx[m], dw[n]))
            exact = Fraction(s, 2 ** (2 * frac)) * Fraction(float(xs[m])) * Fraction(float(ws[n])) + \
                Fraction(float(bv[n]))
            assert out[m, n] == _nearest_bf16(exact)


def test_gemm_bias_special_cases():
    rng = np.random.default_rng(32)
    M, N, K = 3, 8, 16
    wq = _rand_codes(rng, (N, K), O.E4M3)
    xs = np.ones(M, np.float32)
    ws = rng.uniform(0.1, 1, N).astype(np.float32)
    bias = W.f32_to_bf16_bits(rng.standard_normal(N).astype(np.float32))
    bias[0] = 0x8000  # -0.0: -0 + (+0 product) is +0
    # all-zero activations: the output is the bias itself
    out = O.gemm_a8w8_bias(np.zeros((M, K), np.uint8), wq, O.E4M3, xs, ws, bias)
    expect = np.tile(bias, (M, 1))
    expect[:, 0] = 0
    np.testing.assert_array_equal(out, expect)
    # a zero bias gives the plain GEMM
    xq = _rand_codes(rng, (M, K), O.E4M3)
    np.testing.assert_array_equal(O.gemm_a8w8_bias(xq, wq, O.E4M3, xs, ws, np.zeros(N, np.uint16)),
                                  O.gemm_a8w8(xq, wq, O.E4M3, xs, ws))


def test_gemm_entries_match_full():
    rng = np.random.default_rng(4)
    M, N, K = 9, 13, 48
    xq = _rand_codes(rng, (M, K), O.E4M3)
    wq = _rand_codes(rng, (N, K), O.E4M3)
    xs = rng.uniform(0.1, 1, M).astype(np.float32)
    ws = rng.uniform(0.1, 1, N).astype(np.float32)
    full = O.gemm_a8w8(xq, wq, O.E4M3, xs, ws)
    ms = rng.integers(0, M, 30)
    ns = rng.integers(0, N, 30)
    np.testing.assert_array_equal(O.gemm_a8w8_entries(xq, wq, O.E4M3, xs, ws, ms, ns), full[ms, ns])


# ----------------------------------------------------------------- grouped
def test_grouped_a8w8_vs_per_expert_numpy():
    rng = np.random.default_rng(21)
    E, N, K = 5, 16, 64
    off = np.array([0, 3, 3, 10, 10, 17], np.int32)  # experts 1 and 3 empty
    M = int(off[-1])
    xq = _rand_codes(rng, (M, K), O.E4M3)
    wq = _rand_codes(rng, (E, N, K), O.E4M3)
    xs = rng.uniform(0.1, 1, M).astype(np.float32)
    ws = rng.uniform(0.1, 1, (E, N)).astype(np.float32)
    sentinel = np.full((M + 2, N), 0xFFFF, np.uint16)
    out = O.grouped_gemm_a8w8(xq, wq, O.E4M3, xs, ws, off, out=sentinel[:M])
    for e in range(E):
        a, b = off[e], off[e + 1]
        S = xq[a:b].view(ml_dtypes.float8_e4m3fn).astype(np.float64) @ \
            wq[e].view(ml_dtypes.float8_e4m3fn).astype(np.float64).T
        v = xs[a:b, None].astype(np.float64) * ws[e][None, :].astype(np.float64) * S
        exp = np.array([O.double_to_bf16(t) for t in v.reshape(-1)], np.uint16).reshape(v.shape)
        np.testing.assert_array_equal(out[a:b], exp)
    assert (sentinel[M:] == 0xFFFF).all()  # nothing written past M_total
    # overwrite, never accumulate (megablocks-hip TODO-gg.md): a second call
    # into the same buffer gives the same bytes
    out2 = O.grouped_gemm_a8w8(xq, wq, O.E4M3, xs, ws, off, out=out.copy())
    np.testing.assert_array_equal(out2, out)


def test_grouped_rows_outside_experts_untouched_and_bad_offsets():
    rng = np.random.default_rng(22)
    xq = _rand_codes(rng, (4, 32), O.E4M3)
    wq = _rand_codes(rng, (2, 8, 32), O.E4M3)
    xs = np.ones(4, np.float32)
    ws = np.ones((2, 8), np.float32)
    with pytest.raises(ValueError):
        O.grouped_gemm_a8w8(xq, wq, O.E4M3, xs, ws, np.array([0, 3, 2], np.int32))
    with pytest.raises(ValueError):
        O.grouped_gemm_a8w8(xq, wq, O.E4M3, xs, ws, np.array([1, 2, 4], np.int32))


def test_grouped_bf16_vs_exact_fractions():
    rng = np.random.default_rng(23)
    E, N, K = 3, 4, 40
    off = np.array([0, 2, 2, 5], np.int32)
    M = 5
    x = W.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    w = W.f32_to_bf16_bits(rng.standard_normal((E, N, K)).astype(np.float32) * np.float32(0.02))
    out = O.grouped_gemm_bf16(x, w, off)
    xf = W.bf16_bits_to_f32(x)
    wf = W.bf16_bits_to_f32(w)
    for e in range(E):
        for m in range(off[e], off[e + 1]):
            for n in range(N):
                s = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(xf[m], wf[e, n]))
                assert out[m, n] == _nearest_bf16(s)


def test_grouped_bf16_cancellation_case():
    # Large cancelling terms: a plain float64 sum would lose the small term;
    # the oracle's compensated sum keeps it exactly.
    big = W.f32_to_bf16_bits(np.array([2.0 ** 60, 1.0, -(2.0 ** 60)], np.float32))
    x = big.reshape(1, 3)
    w = W.f32_to_bf16_bits(np.ones((1, 1, 3), np.float32))
    out = O.grouped_gemm_bf16(x, w, np.array([0, 1], np.int32))
    assert out[0, 0] == 0x3F80  # exactly 1.0


# ---------------------------------------------------------------- workloads
def test_zipf_counts_recipe():
    c = W.zipf_counts(32768, 62, 1.1)
    assert c.sum() == 32768 and c.max() == 8251 and c.min() == 88
    off = W.moe_offsets()
    cnt = np.diff(off)
    assert off[0] == 0 and off[-1] == 32768 and cnt[7] == 0 and cnt[41] == 0
    assert (cnt == 0).sum() == 2


def test_ring_update_matches_quantize_ring_and_f16_input():
    # ring_update is the ring step of the delayed quantize, exposed alone
    rng = np.random.default_rng(31)
    x = rng.standard_normal((6, 10)).astype(np.float32) * np.float32(7.0)
    r1 = np.array([3.0, 0.5, 2.0, 9.0, 100.0, 0.0], np.float32)
    r2 = r1.copy()
    O.quantize(x, O.E5M2, O.PER_TENSOR, ring=r1, ring_idx=2, ring_margin=1)
    O.ring_update(float(np.abs(x).max()), O.E5M2, r2, 2, 1)
    np.testing.assert_array_equal(r1, r2)
    # float16 input: values widen exactly; codes equal those of the f32 copy
    h = (rng.standard_normal((5, 24)) * 30).astype(np.float16)
    h[0, 0] = np.float16(np.inf)
    h[1, 1] = np.float16(np.nan)
    for gran in (O.PER_TENSOR, O.PER_TOKEN, O.PER_CHANNEL):
        qa, sa, aa = O.quantize(h, O.E4M3, gran)
        qb, sb, ab = O.quantize(h.astype(np.float32), O.E4M3, gran)
        np.testing.assert_array_equal(qa, qb)
        np.testing.assert_array_equal(sa, sb)


# ------------------------------------------------------ stochastic E5M2
def _golden_splitmix():
    rows = []
    for line in open(os.path.join(GOLDEN, "splitmix64.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            seed, idx, out = line.split()
            rows.append((int(seed), int(idx), int(out, 16)))
    return rows


def test_splitmix64_published_outputs():
    rows = _golden_splitmix()
    outs = O.splitmix64_outputs(0, len(rows))
    for (seed, idx, out), got in zip(rows, outs):
        assert got == out
        # the counter form: element idx draws the top half of output idx
        assert O.sr_bits(seed, idx) == out >> 32


def test_sr_grid_values_are_fixed_points():
    # a value already on the E5M2 grid never moves, whatever the draw
    for c in range(256):
        v = O.decode(c, O.E5M2)
        if not np.isfinite(v):
            continue
        for u in (0, 1, 0x7FFFFFFF, 0xFFFFFFFF):
            assert O.encode_e5m2_sr(v, u) == O.encode_sat(np.float32(v), O.E5M2)


def _neighbours(y):
    """The E5M2 values just below and above |y| (same sign) and the exact
    fraction of the way from the lower to the upper one."""
    a = abs(Fraction(float(y)))
    e = math.floor(math.log2(a))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    g = Fraction(2) ** (max(e, -14) - 2)
    lo = (a // g) * g
    return lo, lo + g, (a - lo) / g


def test_sr_rounds_between_neighbours_at_the_exact_threshold():
    rng = np.random.default_rng(5)
    ys = list((rng.standard_normal(300) * np.exp(rng.uniform(-14, 10, 300))).astype(np.float32))
    ys += [np.float32(3e-6), np.float32(-1.7e-5), np.float32(6.1e-5), np.float32(1.5), np.float32(-40000.0)]
    for y in ys:
        if abs(float(y)) >= 57344 or y == 0:
            continue
        lo, hi, frac = _neighbours(y)
        if frac == 0:
            continue
        thr = math.floor(frac * 2 ** 32)  # round up iff u < thr
        sign = -1 if y < 0 else 1
        c_lo = O.encode_sat(np.float32(sign * float(lo)), O.E5M2)
        c_hi = O.encode_sat(np.float32(sign * float(hi)), O.E5M2)
        assert O.encode_e5m2_sr(y, 0) == (c_hi if thr > 0 else c_lo)
        if thr > 0:
            assert O.encode_e5m2_sr(y, thr - 1) == c_hi
        assert O.encode_e5m2_sr(y, min(thr, 2 ** 32 - 1)) == c_lo
        assert O.encode_e5m2_sr(y, 2 ** 32 - 1) == c_lo


def test_sr_special_values():
    assert O.encode_e5m2_sr(np.float32(np.nan), 0) == 0x7F
    for y, u in [(np.inf, 0), (-np.inf, 5), (60000.0, 0), (-57344.0, 1)]:
        assert O.encode_e5m2_sr(np.float32(y), u) == O.encode_sat(np.float32(y), O.E5M2)
    assert O.encode_e5m2_sr(np.float32(0.0), 0) == 0x00
    assert O.encode_e5m2_sr(np.float32(-0.0), 0) == 0x80
    # a negative value rounded down to zero keeps its sign
    assert O.encode_e5m2_sr(np.float32(-1e-9), 0xFFFFFFFF) == 0x80


def test_sr_frequency_matches_the_fraction():
    # over many element indices the up-rounding rate is the fraction (5 sigma),
    # which also makes the rounding unbiased in the mean
    n = 20000
    for y in (np.float32(1.3), np.float32(-0.0021), np.float32(2.5e-5)):
        lo, hi, frac = _neighbours(y)
        sign = -1 if y < 0 else 1
        c_hi = O.encode_sat(np.float32(sign * float(hi)), O.E5M2)
        ups = sum(O.encode_e5m2_sr(y, O.sr_bits(77, i)) == c_hi for i in range(n))
        p = float(frac)
        assert abs(ups / n - p) <= 5 * math.sqrt(p * (1 - p) / n) + 1e-9
        mean = sign * (float(lo) + (ups / n) * float(hi - lo))
        assert abs(mean - float(y)) <= 5 * math.sqrt(p * (1 - p) / n) * float(hi - lo) + 1e-12


def test_sr_quantize_scales_match_and_codes_are_neighbours():
    rng = np.random.default_rng(8)
    x = W.f32_to_bf16_bits(rng.standard_normal((24, 96)).astype(np.float32) * np.float32(3.0))
    for gran in (O.PER_TENSOR, O.PER_TOKEN, O.PER_CHANNEL):
        q, s, a = O.quantize_e5m2_sr(x, gran, seed=1234)
        qr, sr_, ar = O.quantize(x, O.E5M2, gran)
        np.testing.assert_array_equal(s.view(np.uint32), sr_.view(np.uint32))
        np.testing.assert_array_equal(a.view(np.uint32), ar.view(np.uint32))
        # the stochastic code is the RNE code or its neighbour on the other side
        d = O.decode_array(q.reshape(-1), O.E5M2) - O.decode_array(qr.reshape(-1), O.E5M2)
        assert (q != qr).any() and (q == qr).any()
        v = O.decode_array(qr.reshape(-1), O.E5M2)
        assert (np.abs(d) <= np.abs(v) * 0.5 + 2.0 ** -16).all()
        # reproducible by seed, different under another seed
        assert np.array_equal(O.quantize_e5m2_sr(x, gran, seed=1234)[0], q)
        assert not np.array_equal(O.quantize_e5m2_sr(x, gran, seed=99)[0], q)


# ------------------------------------------------------------ block-wise
@pytest.mark.parametrize("fmt", FMTS)
def test_blockwise_reduces_to_per_token_when_one_block_spans_the_row(fmt):
    rng = np.random.default_rng(61)
    x = W.f32_to_bf16_bits(rng.standard_normal((9, 96)).astype(np.float32) * np.float32(7.0))
    q, s, a = O.quantize_blockwise(x, fmt, 96)
    qt, st, at = O.quantize(x, fmt, O.PER_TOKEN)
    np.testing.assert_array_equal(q, qt)
    np.testing.assert_array_equal(s.reshape(-1).view(np.uint32), st.view(np.uint32))
    np.testing.assert_array_equal(a.reshape(-1).view(np.uint32), at.view(np.uint32))
    # a block at least as long as the row behaves the same
    q2, s2, _ = O.quantize_blockwise(x, fmt, 1000)
    np.testing.assert_array_equal(q2, qt)
    assert s2.shape == (9, 1)


def test_blockwise_blocks_are_independent_row_slices():
    # each block equals a per-token quantize of that slice alone; the ragged
    # last block is the short remainder of the row
    rng = np.random.default_rng(62)
    x = (rng.standard_normal((5, 100)) * np.exp(rng.uniform(-3, 3, (5, 100)))).astype(np.float32)
    x[2, 32:64] = 0.0          # an all-zero block: scale 1, codes 0
    x[3, 7] = np.nan
    x[4, 99] = np.inf
    q, s, a = O.quantize_blockwise(x, O.E4M3, 32)
    assert s.shape == (5, 4)
    for b, (c0, c1) in enumerate([(0, 32), (32, 64), (64, 96), (96, 100)]):
        qb, sb, ab = O.quantize(np.ascontiguousarray(x[:, c0:c1]), O.E4M3, O.PER_TOKEN)
        np.testing.assert_array_equal(q[:, c0:c1], qb)
        np.testing.assert_array_equal(s[:, b], sb)
        np.testing.assert_array_equal(a[:, b], ab)
    assert s[2, 1] == 1.0 and (q[2, 32:64] == 0).all()


def test_blockwise_single_element_blocks_hit_the_max_code():
    # block 1: every finite nonzero element is its own amax, so |y| = fmax
    x = np.array([[1.5, -0.25, 3e-5, 0.0, 7.0, -900.0, 1e-30, 2.0]], np.float32)
    q, s, _ = O.quantize_blockwise(x, O.E4M3, 1)
    assert list(q[0]) == [0x7E, 0xFE, 0x7E, 0x00, 0x7E, 0xFE, 0x7E, 0x7E]
    assert s[0, 3] == 1.0


def test_blockwise_stochastic_matches_the_element_rule():
    rng = np.random.default_rng(63)
    x = (rng.standard_normal((3, 64)) * np.float32(5e-3)).astype(np.float32)
    q, s, _ = O.quantize_blockwise(x, O.E5M2, 16, stochastic=True, seed=9)
    for r in range(3):
        for c in range(64):
            y = np.float32(x[r, c] * np.float32(O.multiplier(float(np.abs(x[r, (c // 16) * 16:(c // 16 + 1) * 16]).max()), O.E5M2)))
            assert q[r, c] == O.encode_e5m2_sr(y, O.sr_bits(9, r * 64 + c))
    with pytest.raises(ValueError):
        O.quantize_blockwise(x, O.E4M3, 16, stochastic=True)


def test_blockwise_dequantize_closed_forms():
    rng = np.random.default_rng(64)
    q = rng.integers(0, 256, (4, 48), dtype=np.uint8)
    q[O.decode_array(q.reshape(-1), O.E4M3).reshape(q.shape) != O.decode_array(q.reshape(-1), O.E4M3).reshape(q.shape)] = 0
    sc = np.array([[0.5, 2.0, 0.125]] * 4, np.float32)
    out = O.dequantize_blockwise(q, O.E4M3, 16, sc)
    dec = O.decode_array(q.reshape(-1), O.E4M3).reshape(q.shape)
    np.testing.assert_array_equal(out, (dec * np.repeat(sc, 16, axis=1)).astype(np.float32))  # powers of two: exact
    # bf16 output: the f32 product rounded once
    outb = O.dequantize_blockwise(q, O.E4M3, 16, sc, bf16=True)
    np.testing.assert_array_equal(outb, W.f32_to_bf16_bits(out))
    # a round trip through quantize recovers every value to within half a code step
    x = (rng.standard_normal((4, 48)) * 3).astype(np.float32)
    qq, ss, _ = O.quantize_blockwise(x, O.E4M3, 16)
    back = O.dequantize_blockwise(qq, O.E4M3, 16, ss)
    assert (np.abs(back - x) <= np.abs(x) * 2.0 ** -4 + np.repeat(ss, 16, axis=1) * 2.0 ** -9).all()


# ------------------------------------------------------- block-scaled GEMM
def _exact_block_dot(xq, wq, fmt, k0, k1):
    frac = 9 if fmt == O.E4M3 else 16
    dx = xq.view(ML[fmt]).astype(np.float64)
    dw = wq.view(ML[fmt]).astype(np.float64)
    return Fraction(sum(int(a * 2 ** frac) * int(b * 2 ** frac) for a, b in zip(dx[k0:k1], dw[k0:k1])),
                    2 ** (2 * frac))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("block", [16, 32, 48])
def test_blockscaled_gemm_vs_fractions(fmt, block):
    # sum over blocks of xs[m,b] ws[n,b] S_b in exact rationals, the last block
    # the short remainder of K (K = 80), one round to nearest-even bf16
    rng = np.random.default_rng(70 + block + fmt)
    M, N, K = 5, 7, 80
    nb = -(-K // block)
    xq = _rand_codes(rng, (M, K), fmt)
    wq = _rand_codes(rng, (N, K), fmt)
    xs = rng.uniform(1e-3, 4, (M, nb)).astype(np.float32)
    ws = rng.uniform(1e-3, 4, (N, nb)).astype(np.float32)
    bias = W.f32_to_bf16_bits(rng.standard_normal(N).astype(np.float32))
    out = O.gemm_blockscaled(xq, wq, fmt, xs, ws, block)
    outb = O.gemm_blockscaled(xq, wq, fmt, xs, ws, block, bias)
    bv = W.bf16_bits_to_f32(bias)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(xs[m, b])) * Fraction(float(ws[n, b])) *
                        _exact_block_dot(xq[m], wq[n], fmt, b * block, min(K, (b + 1) * block)) for b in range(nb))
            assert out[m, n] == _nearest_bf16(exact)
            assert outb[m, n] == _nearest_bf16(exact + Fraction(float(bv[n])))


@pytest.mark.parametrize("fmt", FMTS)
def test_blockscaled_gemm_one_block_is_the_scaled_gemm(fmt):
    # a block spanning K leaves one scale per row and per column: the per-row /
    # per-column scaled GEMM (and its bias form), bit for bit
    rng = np.random.default_rng(75)
    M, N, K = 6, 9, 64
    xq = _rand_codes(rng, (M, K), fmt)
    wq = _rand_codes(rng, (N, K), fmt)
    xs = rng.uniform(0.01, 3, (M, 1)).astype(np.float32)
    ws = rng.uniform(0.01, 3, (N, 1)).astype(np.float32)
    bias = W.f32_to_bf16_bits(rng.standard_normal(N).astype(np.float32))
    for block in (64, 128, 4096):
        assert np.array_equal(O.gemm_blockscaled(xq, wq, fmt, xs, ws, block), O.gemm_a8w8(xq, wq, fmt, xs, ws))
        assert np.array_equal(O.gemm_blockscaled(xq, wq, fmt, xs, ws, block, bias),
                              O.gemm_a8w8_bias(xq, wq, fmt, xs, ws, bias))


def test_blockscaled_gemm_uniform_power_of_two_scales():
    # with the same power-of-two scale in every block of a row (and of a
    # column) every step is exact, so the blocks sum to the unblocked GEMM
    rng = np.random.default_rng(76)
    M, N, K, block = 8, 12, 96, 32
    xq = _rand_codes(rng, (M, K), O.E4M3)
    wq = _rand_codes(rng, (N, K), O.E4M3)
    xs1 = (2.0 ** rng.integers(-6, 6, M)).astype(np.float32)
    ws1 = (2.0 ** rng.integers(-6, 6, N)).astype(np.float32)
    xs = np.repeat(xs1[:, None], K // block, axis=1)
    ws = np.repeat(ws1[:, None], K // block, axis=1)
    assert np.array_equal(O.gemm_blockscaled(xq, wq, O.E4M3, xs, ws, block), O.gemm_a8w8(xq, wq, O.E4M3, xs1, ws1))


def test_blockscaled_gemm_blocks_are_separate_terms():
    # codes zero outside block 1 leave only that block's term; doubling the
    # x scale of a block whose codes are all zero changes nothing
    rng = np.random.default_rng(77)
    M, N, K, block = 4, 5, 96, 32
    xq = _rand_codes(rng, (M, K), O.E4M3)
    wq = _rand_codes(rng, (N, K), O.E4M3)
    xq[:, :block] = 0
    xq[:, 2 * block:] = 0
    xs = rng.uniform(0.1, 2, (M, 3)).astype(np.float32)
    ws = rng.uniform(0.1, 2, (N, 3)).astype(np.float32)
    got = O.gemm_blockscaled(xq, wq, O.E4M3, xs, ws, block)
    one = O.gemm_a8w8(np.ascontiguousarray(xq[:, block:2 * block]), np.ascontiguousarray(wq[:, block:2 * block]),
                      O.E4M3, xs[:, 1], ws[:, 1])
    assert np.array_equal(got, one)
    xs2 = xs.copy()
    xs2[:, 0] *= 2
    assert np.array_equal(O.gemm_blockscaled(xq, wq, O.E4M3, xs2, ws, block), got)


def test_blockscaled_gemm_entries_equal_the_full_product():
    rng = np.random.default_rng(78)
    M, N, K, block = 9, 11, 144, 64
    xq = _rand_codes(rng, (M, K), O.E5M2)
    wq = _rand_codes(rng, (N, K), O.E5M2)
    xs = rng.uniform(0.1, 2, (M, 3)).astype(np.float32)
    ws = rng.uniform(0.1, 2, (N, 3)).astype(np.float32)
    bias = W.f32_to_bf16_bits(rng.standard_normal(N).astype(np.float32))
    full = O.gemm_blockscaled(xq, wq, O.E5M2, xs, ws, block, bias)
    ms = rng.integers(0, M, 30)
    ns = rng.integers(0, N, 30)
    assert np.array_equal(O.gemm_blockscaled_entries(xq, wq, O.E5M2, xs, ws, block, ms, ns, bias), full[ms, ns])


@pytest.mark.parametrize("fmt,rel,sub", [(O.E4M3, 2.0 ** -4, 2.0 ** -10), (O.E5M2, 2.0 ** -3, 2.0 ** -17)])
def test_blockwise_round_trip_within_half_a_step(fmt, rel, sub):
    # decode(quantize(x)) * block scale is within half a code step of x:
    # 2^-(mantissa bits + 1) relative for normal codes, half the subnormal
    # step (scaled) otherwise; a block index mixed up between the two
    # functions breaks it at once
    rng = np.random.default_rng(79)
    rows, cols, block = 6, 200, 32
    band = np.exp(rng.uniform(-10, 6, (rows, -(-cols // 8)))).repeat(8, axis=1)[:, :cols]
    x = (rng.standard_normal((rows, cols)) * band).astype(np.float32)
    q, s, _ = O.quantize_blockwise(x, fmt, block)
    back = O.dequantize_blockwise(q, fmt, block, s).astype(np.float64)
    sc = np.repeat(s, block, axis=1)[:, :cols].astype(np.float64)
    err = np.abs(back - x.astype(np.float64))
    assert (err <= np.abs(x) * (rel + 2.0 ** -20) + sc * sub).all()


# ------------------------------------------------------------ bias gradient
# AstrAI ops.cu linear_backward_fp8: the bias gradient is g summed over dim 0
# and cast back to g's dtype.


def test_double_to_f16_matches_numpy():
    # the oracle's own f16 rounding against numpy's double -> half cast (an
    # independent implementation), over 12 decades and the edges: the largest
    # finite value, the overflow threshold 65520, subnormals, signed zero, Inf
    rng = np.random.default_rng(91)
    v = rng.standard_normal(20000) * np.exp(rng.uniform(-25, 12, 20000))
    v = np.concatenate([v, [65504.0, 65519.99, 65520.0, -65520.0, 1e-8, 6e-8, 2.98e-8, -0.0, 0.0,
                            np.inf, -np.inf, 2.0 ** -24 * 1.5, 2.0 ** -14 * (1 - 2.0 ** -11)]])
    mine = np.array([O.double_to_f16(float(x)) for x in v], np.uint16)
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).view(np.uint16)
    assert np.array_equal(mine, ref)
    assert O.double_to_f16(float("nan")) & 0x7C00 == 0x7C00 and O.double_to_f16(float("nan")) & 0x3FF


def test_grad_bias_closed_form():
    # g[r, c] = (r + 1) * (c % 5 - 2): the column sums are (c % 5 - 2) * R(R+1)/2,
    # exact in every dtype for R = 15 (120 * 2 = 240 < 256); a transposed or
    # shifted index changes them
    R, C = 15, 37
    r = np.arange(1, R + 1, dtype=np.float64)[:, None]
    c = (np.arange(C) % 5 - 2).astype(np.float64)[None, :]
    g = r * c
    want = (np.arange(C) % 5 - 2) * (R * (R + 1) // 2)
    out32 = O.grad_bias(g.astype(np.float32))
    assert np.array_equal(out32, want.astype(np.float32))
    out16 = O.grad_bias(g.astype(np.float16))
    assert np.array_equal(out16.astype(np.float64), want)
    outb = O.grad_bias(W.f32_to_bf16_bits(g.astype(np.float32)))
    assert np.array_equal(O.bf16_bits_to_f32(outb).astype(np.float64), want)
    assert O.grad_bias(np.zeros((0, 4), np.float32)).tolist() == [0.0] * 4


def test_grad_bias_is_the_rounded_exact_sum():
    # random bf16 g: the fp64 sums (exact here: 300 terms of 8-bit
    # significands within 2^40 of each other) against an exact integer
    # re-summation, and the output is that sum rounded once to bf16
    rng = np.random.default_rng(92)
    R, C = 300, 41
    x = (rng.standard_normal((R, C)) * 3).astype(np.float32)
    x[np.abs(x) < 2.0 ** -30] = 0.0  # every value a multiple of 2^-40 after bf16 rounding
    gb = W.f32_to_bf16_bits(x)
    out, ref = O.grad_bias(gb, return_ref=True)
    vals = O.bf16_bits_to_f32(gb).astype(np.float64)
    scale = 2.0 ** 40
    exact = (vals * scale).astype(np.int64).sum(axis=0) / scale  # integers: exact
    assert np.array_equal(ref, exact)
    assert np.array_equal(out, np.array([O.double_to_bf16(v) for v in exact], np.uint16))


def test_grad_bias_non_finite():
    g = np.ones((6, 4), np.float32)
    g[2, 1] = np.nan
    g[3, 2] = np.inf
    g[1, 3], g[4, 3] = np.inf, -np.inf
    out = O.grad_bias(g)
    assert out[0] == 6.0 and np.isnan(out[1]) and out[2] == np.inf and np.isnan(out[3])
