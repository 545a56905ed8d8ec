"""Pins for the oracle's FP4 E2M1 / E4M3 number formats and FP4 quantizer.

The oracle's encoders search the value set by distance; here they are checked
against an independent implementation (the ml_dtypes format library), against
closed forms of the formats, and against the invariants that the FP4 scheme
implies (exact round trips, power-of-two scale shifts, sign symmetry, error
bounds, 288 bytes per 512-channel token).
"""
import os
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_e2m1():
    rows = []
    for line in open(os.path.join(GOLDEN, "e2m1_values.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        c, v = line.split()
        rows.append((int(c), float(v)))
    return rows


def test_e2m1_value_table_matches_golden_and_library():
    rows = _golden_e2m1()
    assert [c for c, _ in rows] == list(range(16))
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    for c, v in rows:
        got = oracle.e2m1_value(c)
        assert got == v and np.signbit(got) == np.signbit(v), (c, got, v)
        assert got == lib[c] and np.signbit(got) == np.signbit(lib[c])
    mags = sorted({abs(v) for _, v in rows})
    assert mags == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e4m3_decode_all_codes_closed_form_and_library():
    lib = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for c in range(256):
        v = oracle.e4m3_value(c)
        if c in (0x7F, 0xFF):
            assert np.isnan(v) and np.isnan(lib[c])
            continue
        assert v == lib[c], (c, v, lib[c])
        # closed form: sign * 2^(e-7) * (1 + m/8), subnormal m * 2^-9
        s, e, m = c >> 7, (c >> 3) & 15, c & 7
        ref = Fraction(m, 512) if e == 0 else Fraction(8 + m, 8) * Fraction(2) ** (e - 7)
        assert Fraction(abs(v)) == ref
        assert np.signbit(v) == bool(s)
    assert oracle.e4m3_value(0x7E) == 448.0
    assert oracle.e4m3_value(0x01) == 2.0 ** -9


def _probe_values():
    """fp32 probes: every exponent from 2^-30 to 2^12 with a spread of
    mantissas, plus +-4 ulps around every E2M1 value, every E2M1 tie point and
    every E4M3 value / tie point, plus zeros, subnormals and huge values."""
    rng = np.random.default_rng(1234)
    out = []
    exps = np.arange(127 - 30, 127 + 13, dtype=np.uint32)
    mant = np.concatenate([np.arange(0, 1 << 23, 997, dtype=np.uint32),
                           np.array([0, 1, 2, (1 << 22), (1 << 23) - 1], np.uint32)])
    bits = (exps[:, None] << 23) | mant[None, :]
    out.append(bits.ravel().view(np.float32))
    pts = [0.0, 0.25, 0.5, 0.75, 1.0, 1.25, 1.5, 1.75, 2.0, 2.5, 3.0, 3.5, 4.0, 5.0, 6.0, 7.0]
    e4 = np.arange(0x7F, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    mids = (e4[1:] + e4[:-1]) / 2
    pts += list(e4) + list(mids) + [464.0, 480.0]
    for p in pts:
        f = np.float32(p)
        b = np.array([f], np.float32).view(np.uint32)[0]
        for d in range(-4, 5):
            if int(b) + d >= 0:
                out.append(np.array([int(b) + d], np.uint32).view(np.float32))
    out.append(np.array([0.0, 1e-45, 1e-40, 1.17e-38, 1e-10, 1e6, 1e30, 3.4e38], np.float32))
    out.append(rng.standard_normal(20000).astype(np.float32) * 3)
    v = np.concatenate(out).astype(np.float32)
    return np.concatenate([v, -v])


def test_e2m1_encode_matches_library_round_to_nearest_even_saturating():
    v = _probe_values()
    got = oracle.e2m1_encode_array(v)
    ref = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(v[i]), int(got[i]), int(ref[i])) for i in bad[:10]]


def test_e2m1_tie_and_saturation_cases():
    # ties go to the even code; above 6 saturates; the sign survives rounding to 0
    cases = [(0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6), (6.5, 7),
             (1e9, 7), (0.2500001, 1), (0.2499999, 0), (-0.1, 8), (-0.0, 8), (0.0, 0)]
    for x, code in cases:
        assert oracle.e2m1_encode(x) == code, (x, oracle.e2m1_encode(x), code)


def test_e4m3_encode_matches_library_in_range_and_saturates_above():
    v = _probe_values()
    got = oracle.e4m3_encode_array(v)
    inr = np.abs(v) < 464.0      # ml_dtypes rounds values >= 464 to NaN (no saturation)
    ref = v[inr].astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    bad = np.nonzero(got[inr] != ref)[0]
    assert bad.size == 0, [(float(v[inr][i]), int(got[inr][i]), int(ref[i])) for i in bad[:10]]
    sat = got[~inr]
    assert np.all((sat & 0x7F) == 0x7E)


def _trunc_bf16(x):
    """float32 array -> bf16 bit patterns by dropping the low 16 bits."""
    return (np.ascontiguousarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _bf16(x):
    """float32 array -> bf16 bit patterns (x must be exactly representable)."""
    u = np.asarray(x, np.float32).view(np.uint32)
    assert np.all((u & 0xFFFF) == 0)
    return (u >> 16).astype(np.uint16)


def test_quantize_exact_round_trip():
    rng = np.random.default_rng(7)
    e2m1 = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float64)
    e4 = np.arange(0x7F, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for _ in range(200):
        sc = int(rng.integers(0x08, 0x7F))      # normal-range scale codes
        s = e4[sc]
        k = rng.choice(e2m1, 16) * rng.choice([-1, 1], 16)
        k[rng.integers(16)] = 6.0 * rng.choice([-1, 1])   # amax = 6 s, so amax/6 = s exactly
        x = (k * s).astype(np.float32)
        if not np.all((x.view(np.uint32) & 0xFFFF) == 0):
            continue                                 # not representable in bf16
        packed, sf = oracle.fp4_quantize(_bf16(x)[None, :])
        assert sf[0, 0] == sc
        back = oracle.fp4_dequantize(packed, sf)[0]
        assert np.array_equal(back, k * s)


def test_quantize_power_of_two_scale_shift_and_negation():
    rng = np.random.default_rng(11)
    x = rng.standard_normal((64, 64)).astype(np.float32)
    xb = _trunc_bf16(x)
    base = np.asarray(xb.astype(np.uint32) << 16).view(np.float32)
    p0, s0 = oracle.fp4_quantize(xb)
    for e in (-3, -1, 1, 2):
        p1, s1 = oracle.fp4_quantize(_bf16(base * np.float32(2.0 ** e)))
        assert np.array_equal(p0, p1)
        assert np.array_equal(s1.astype(int) - s0.astype(int), np.full(s0.shape, 8 * e))
    pn, sn = oracle.fp4_quantize(_bf16(-base))
    assert np.array_equal(sn, s0)
    # negation flips only the sign bit of each nibble (entries that round to 0 keep
    # their magnitude code 0 and get the opposite sign bit)
    assert np.array_equal(pn ^ p0, np.full(p0.shape, 0x88, np.uint8))


def test_quantize_error_bound_and_zero_group():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((256, 128)) * rng.choice([1, 8], 128)).astype(np.float32)
    xb = _trunc_bf16(x)
    xv = np.asarray(xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    packed, sf = oracle.fp4_quantize(xb)
    back = oracle.fp4_dequantize(packed, sf)
    scale = sf.view(ml_dtypes.float8_e4m3fn).astype(np.float64).repeat(16, axis=1)
    v = np.abs(xv) / scale
    err = np.abs(xv - back)
    # E2M1 spacing: 0.5 below 2, 1 in [2, 4), 2 in [4, 6]; saturation adds at most
    # (6.4 - 6) s because the E4M3 rounding of amax/6 is within 2^-4 relative.
    bound = np.where(v < 2, 0.25, np.where(v < 4, 0.5, 1.0)) * scale
    assert np.all(err <= bound + 1e-12)
    # all-zero group: scale code 0 and all codes +0
    z = np.zeros((1, 32), np.uint16)
    p, s = oracle.fp4_quantize(z)
    assert np.all(p == 0) and np.all(s == 0)
    # a group of negative zeros: its scale is 0, so every code is +0 (no sign kept)
    nz = np.full((1, 16), 0x8000, np.uint16)
    p, s = oracle.fp4_quantize(nz)
    assert np.all(p == 0) and np.all(s == 0)
    # a group whose amax/6 rounds below the smallest E4M3 subnormal: scale 0, codes +0
    tiny = _bf16(np.full(16, 2.0 ** -13, np.float32))[None, :]
    p, s = oracle.fp4_quantize(tiny)
    assert s[0, 0] == 0 and np.all(p == 0)


def _nvfp4_pack_restated(x_bf16):
    """The FP4 pack of [N] "FP4 KV Quantization and Cache Lifetime Management"
    (E2M1 elements, one E4M3 scale per 16 channels, NVFP4 without its global
    scale) restated with numpy float32 arithmetic and the ml_dtypes format
    casts, sharing nothing with the oracle's C code: per group amax, then
    s_f = float32(amax) / float32(6) (IEEE division), scale = E4M3 RNE of s_f
    saturating at 448, each element float32(x) / float32(scale) (IEEE
    division) cast to E2M1 (RNE, saturating, sign kept), a zero scale giving
    +0 codes, two codes per byte with the even channel in the low nibble."""
    x = np.ascontiguousarray(x_bf16, np.uint16)
    rows, C = x.shape
    xf = (x.astype(np.uint32) << 16).view(np.float32).reshape(rows, C // 16, 16)
    amax = np.abs(xf).max(axis=2)
    s_f = amax / np.float32(6)
    assert s_f.dtype == np.float32
    s_code = np.minimum(s_f, np.float32(448)).astype(ml_dtypes.float8_e4m3fn)
    s = s_code.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = xf / s[:, :, None]
    assert v.dtype == np.float32
    codes = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    codes = np.where(s[:, :, None] == 0, np.uint8(0), codes).reshape(rows, C)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, s_code.view(np.uint8)


def _tie_multiple_groups():
    """One group per (E4M3 scale s, E2M1 tie point k): an element 6 s (so amax/6
    is exactly s) and the others k s for the seven ties k = 0.25 ... 5 with both
    signs, all exactly representable in bf16. x / s is then exactly the tie; a
    division that is off by one ulp breaks it the other way."""
    e4 = np.arange(1, 0x7F, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    groups = []
    for s in e4:
        for lead in (1.0, -1.0):
            g = np.concatenate([[6.0 * lead], ties, -ties, [0.0]]) * s
            groups.append(g)
    x = np.array(groups, np.float32)
    return _bf16(x)


def _scale_midpoint_groups():
    """Groups whose amax / 6 is exactly the midpoint of two neighbouring E4M3
    values (a tie of the scale rounding), with tie-multiple elements of the
    scale that the midpoint rounds to."""
    e4 = np.arange(0, 0x7F, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    mids = (e4[1:] + e4[:-1]) / 2
    out = []
    for m in mids:
        amax = 6.0 * m
        if amax > 3.0e38:
            continue
        body = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 1.5, 3.0, 4.0, 6.0, 2.0, 1.0, 0.0]) * m
        for sign in (1.0, -1.0):
            out.append(np.concatenate([[sign * amax], body * sign]))
    x = np.array(out, np.float32)
    u = x.view(np.uint32)
    keep = np.all((u & 0xFFFF) == 0, axis=1)       # every value exact in bf16
    return (u[keep] >> 16).astype(np.uint16)


def _random_finite_bf16_groups(n_groups, seed):
    rng = np.random.default_rng(seed)
    x = rng.integers(0, 1 << 16, size=(n_groups, 16), dtype=np.uint32).astype(np.uint16)
    finite = (x & 0x7F80) != 0x7F80
    return np.where(finite, x, np.uint16(0)).astype(np.uint16)


@pytest.mark.parametrize("inputs", ["tie_multiples", "scale_midpoints", "random_bits"])
def test_quantize_matches_independent_nvfp4_restatement(inputs):
    if inputs == "tie_multiples":
        x = _tie_multiple_groups()
        assert x.shape[0] == 2 * 126
    elif inputs == "scale_midpoints":
        x = _scale_midpoint_groups()
        assert x.shape[0] >= 200
    else:
        x = _random_finite_bf16_groups(262_144, seed=29)
    # rows of 16 groups (256 channels) keep the layout of a real cache row
    pad = (-x.shape[0]) % 16
    x = np.concatenate([x, np.zeros((pad, 16), np.uint16)]).reshape(-1, 256)
    packed, sf = oracle.fp4_quantize(x)
    rp, rs = _nvfp4_pack_restated(x)
    bad_s = np.argwhere(sf != rs)
    assert bad_s.size == 0, bad_s[:5]
    bad_p = np.argwhere(packed != rp)
    assert bad_p.size == 0, [(tuple(i), int(packed[tuple(i)]), int(rp[tuple(i)])) for i in bad_p[:5]]


def every_bf16_amax_groups():
    """One 16-channel group per finite bf16 magnitude a (both signs): a in
    channel 0, a/2 rounded down to bf16 in channel 1, zeros elsewhere. The
    group's amax runs over every finite bf16 value."""
    b = np.arange(1, 0x7F80, dtype=np.uint16)
    g = np.zeros((2 * b.size, 16), np.uint16)
    g[:b.size, 0] = b
    g[b.size:, 0] = b | 0x8000
    half = _trunc_bf16(((b.astype(np.uint32) << 16).view(np.float32) / np.float32(2)))
    g[:b.size, 1] = half
    g[b.size:, 1] = half | 0x8000
    return g


def test_quantize_scale_for_every_bf16_amax():
    """The scale step alone, exhaustively: for every finite bf16 amax the
    oracle's scale byte is E4M3_RNE_satfinite(float32(amax) / 6)."""
    g = every_bf16_amax_groups()
    _, sf = oracle.fp4_quantize(g)
    a = np.abs((g[:, 0].astype(np.uint32) << 16).view(np.float32))
    ref = np.minimum(a / np.float32(6), np.float32(448)).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    bad = np.nonzero(sf[:, 0] != ref)[0]
    assert bad.size == 0, [(float(a[i]), int(sf[i, 0]), int(ref[i])) for i in bad[:5]]
    rp, rs = _nvfp4_pack_restated(g)
    assert np.array_equal(rs[:, 0], sf[:, 0])


def test_dequantize_every_code_and_scale_is_exact_product():
    codes = np.arange(16, dtype=np.uint8)
    packed = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)
    for sc in range(0x7F):
        sf = np.array([[sc]], np.uint8)
        out = oracle.fp4_dequantize(packed[None, :], sf)[0]
        s = Fraction(oracle.e4m3_value(sc))
        for c in range(16):
            ref = Fraction(float(np.uint8(c).view(ml_dtypes.float4_e2m1fn).astype(np.float64))) * s
            assert Fraction(out[c]) == ref


def test_fp4_row_bytes_match_pages():
    vals = dict(line.split()[:2] for line in open(os.path.join(GOLDEN, "csa2_layout.txt"))
                if line.strip() and not line.startswith("#"))
    assert oracle.fp4_row_bytes(512) == int(vals["fp4_row_bytes_512"]) == 288
    packed, sf = oracle.fp4_quantize(np.zeros((3, 512), np.uint16))
    assert packed.shape[1] + sf.shape[1] == 288


# ----------------------------------------------------------------------------- MXFP4 variant
# [T] mechanism 3 names the cache format MXFP4; read as the OCP Microscaling
# format: E2M1 elements, one E8M0 scale per 32 channels, shared exponent
# floor(log2(amax)) - 2.
def _trunc_bits(x):
    """float32 values -> bf16 bit patterns (as uint32) by dropping the low 16 bits."""
    return np.asarray(x, dtype=np.float32).view(np.uint32) >> 16


def _floor_log2(x: float) -> int:
    """floor(log2(x)) of a positive float by exact integer arithmetic."""
    n, d = Fraction(x).as_integer_ratio()
    k = n.bit_length() - d.bit_length()
    return k if (Fraction(n, d) >= Fraction(2) ** k) else k - 1


def test_e8m0_decode_all_codes_closed_form_and_library():
    lib = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    for c in range(255):
        v = oracle.e8m0_value(c)
        assert v == lib[c] and Fraction(v) == Fraction(2) ** (c - 127), c
    assert np.isnan(oracle.e8m0_value(255)) and np.isnan(lib[255])


def test_mx_shared_exponent_closed_form():
    rng = np.random.default_rng(21)
    vals = list(2.0 ** rng.uniform(-140, 127, 3000)) + [1.0, 6.0, 7.99, 8.0, 0.25, 2.0 ** -126,
                                                       2.0 ** -149, 3.0e38]
    for amax in vals:
        amax = float(np.float32(amax))
        if amax == 0.0:
            continue
        ref = min(127, max(-127, _floor_log2(amax) - 2))
        assert oracle.mx_shared_exp(amax) == ref, amax
    assert oracle.mx_shared_exp(0.0) == -127
    assert oracle.mx_shared_exp(6.0) == 0 and oracle.mx_shared_exp(1.0) == -2
    assert oracle.mx_shared_exp(7.99) == 0 and oracle.mx_shared_exp(8.0) == 1


def test_mxfp4_quantize_is_e2m1_of_the_scaled_block():
    """Scale codes from the exact exponent of each block's amax; element codes
    from the (library-pinned) E2M1 encoder of x / 2^e; packing low nibble first."""
    rng = np.random.default_rng(22)
    x = (rng.standard_normal((40, 128)) * np.exp(rng.uniform(-20, 20, (40, 1)))).astype(np.float32)
    x[3, :32] = 0.0
    x[5, 40:48] *= 1e4
    xb = _trunc_bits(x).astype(np.uint16)
    xf = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    packed, sf = oracle.mxfp4_quantize(xb)
    for r in range(x.shape[0]):
        for g in range(4):
            blk = xf[r, 32 * g:32 * g + 32]
            amax = float(np.abs(blk).max())
            e = -127 if amax == 0 else min(127, max(-127, _floor_log2(amax) - 2))
            assert sf[r, g] == e + 127
            codes = oracle.e2m1_encode_array((blk / 2.0 ** e).astype(np.float32))
            got = np.stack([packed[r, 16 * g:16 * g + 16] & 15, packed[r, 16 * g:16 * g + 16] >> 4], 1)
            assert np.array_equal(got.ravel(), codes), (r, g)


def test_mxfp4_exact_round_trip_and_invariants():
    rng = np.random.default_rng(23)
    e2m1 = np.array([oracle.e2m1_value(c) for c in range(16)])
    for _ in range(50):
        s = int(rng.integers(-120, 120))
        codes = rng.integers(0, 16, 32)
        codes[rng.integers(0, 32)] = 6 + int(rng.integers(0, 2))   # amax in [4, 6]
        x = e2m1[codes] * 2.0 ** s
        xb = _trunc_bits(x).astype(np.uint16)
        packed, sf = oracle.mxfp4_quantize(xb[None])
        assert sf[0, 0] == s + 127
        assert np.array_equal(oracle.mxfp4_dequantize(packed, sf)[0], x)
        # scaling by 2^t shifts only the scale code; negation flips only the signs
        t = int(rng.integers(-5, 5))
        p2, sf2 = oracle.mxfp4_quantize(_trunc_bits(x * 2.0 ** t).astype(np.uint16)[None])
        assert int(sf2[0, 0]) == int(sf[0, 0]) + t and np.array_equal(p2, packed)
        p3, sf3 = oracle.mxfp4_quantize(_trunc_bits(-x).astype(np.uint16)[None])
        assert np.array_equal(sf3, sf)
        assert np.all((p3 ^ packed) == 0x88)  # every sign bit flips (zeros too)


def test_mxfp4_error_bound_saturation_and_zero_block():
    rng = np.random.default_rng(24)
    x = rng.standard_normal((64, 64)).astype(np.float32) * 3.0
    xb = _trunc_bits(x).astype(np.uint16)
    xf = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    packed, sf = oracle.mxfp4_quantize(xb)
    xh = oracle.mxfp4_dequantize(packed, sf)
    scale = np.repeat(2.0 ** (sf.astype(np.float64) - 127), 32, axis=1)
    v = np.abs(xf) / scale
    err = np.abs(xf - xh) / scale
    # spacing of E2M1 is 0.5 below 2, 1 below 4, 2 below 6; |v| < 8 saturates at 6
    assert np.all(v < 8)
    assert np.all(err[v <= 2] <= 0.25) and np.all(err[(v > 2) & (v <= 4)] <= 0.5)
    assert np.all(err[(v > 4) & (v <= 6)] <= 1.0) and np.all(err[v > 6] <= 2.0)
    z, zs = oracle.mxfp4_quantize(np.zeros((1, 32), np.uint16))
    assert zs[0, 0] == 0 and np.all(z == 0) and np.all(oracle.mxfp4_dequantize(z, zs) == 0)


def test_mxfp4_dequantize_every_code_and_scale_is_exact_product():
    codes = np.arange(16, dtype=np.uint8)
    packed = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)
    packed = np.tile(packed, 4)[None]                      # 32 channels
    for e in range(255):
        out = oracle.mxfp4_dequantize(packed, np.array([[e]], np.uint8))[0]
        for c in range(32):
            assert Fraction(out[c]) == Fraction(oracle.e2m1_value(c % 16)) * Fraction(2) ** (e - 127)


def test_mxfp4_row_bytes():
    # 512 channels: 256 bytes of E2M1 codes + 16 E8M0 scales
    packed, sf = oracle.mxfp4_quantize(np.zeros((1, 512), np.uint16))
    assert packed.shape[-1] + sf.shape[-1] == 272
