"""Pins for the oracle's number formats (CPU only).

BF16 and E4M3 encoders are checked against torch's casts (an independent
library routine) and against exact rational rounding with Python fractions;
the E4M3 decode table against the format definition.
"""
import math
import struct
from fractions import Fraction

import numpy as np
import torch

from oracle import numerics as nm

GOLDEN = __import__("os").path.join(__import__("os").path.dirname(__file__), "golden")


def _f32_bits(v: float) -> int:
    return struct.unpack("<I", struct.pack("<f", v))[0]


def _exact_rne(x: Fraction, unit: Fraction) -> Fraction:
    return Fraction(round(x / unit)) * unit  # Python rounds Fraction halves to even


def _exact_bf16_bits(x: float) -> int:
    """Reference: RNE of the exact value of x onto the BF16 grid."""
    if x == 0.0:
        return 0x8000 if math.copysign(1.0, x) < 0 else 0
    fx = Fraction(x)
    ax = abs(fx)
    E = math.floor(math.log2(abs(x)))
    while Fraction(2) ** E > ax:
        E -= 1
    while Fraction(2) ** (E + 1) <= ax:
        E += 1
    E = max(E, -126)
    q = _exact_rne(ax, Fraction(2) ** (E - 7))
    if q >= Fraction(2) ** 128:
        mag = 0x7F80
    else:
        mag = _f32_bits(float(q)) >> 16
    return mag | (0x8000 if x < 0 else 0)


def test_bf16_widening_roundtrip_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = nm.bf16_bits_to_f32(bits)
    back = nm.f32_to_bf16_bits(f)
    finite = ~np.isnan(f)
    assert np.array_equal(back[finite], bits[finite])
    assert np.all(np.isnan(nm.bf16_bits_to_f32(back[~finite])))


def test_f32_to_bf16_matches_torch():
    hi = np.arange(65536, dtype=np.uint64)
    rng = np.random.default_rng(5)
    lows = np.concatenate([np.array([0, 1, 0x7FFF, 0x8000, 0x8001, 0xFFFF, 0x7FFE, 0x4000]),
                           rng.integers(0, 65536, 24)]).astype(np.uint64)
    u = ((hi[:, None] << np.uint64(16)) | lows[None, :]).ravel().astype(np.uint32)
    x = u.view(np.float32)
    ours = nm.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    fin = ~np.isnan(x)
    assert np.array_equal(ours[fin], ref[fin])


def test_f64_to_bf16_single_rounding_matches_exact():
    rng = np.random.default_rng(6)
    xs = list(rng.standard_normal(3000) * np.exp2(rng.integers(-140, 130, 3000)))
    # exact midpoints between neighbouring BF16 values, and +-1 FP64 ulp around them:
    # a FP64->FP32->BF16 double rounding gets the +-ulp cases wrong.
    for e in (-130, -127, -126, -20, -1, 0, 1, 7, 100, 127):
        for m in (128, 129, 200, 255):
            mid = (m + 0.5) * 2.0 ** (e - 7)
            for v in (mid, np.nextafter(mid, 0), np.nextafter(mid, np.inf)):
                xs += [v, -v]
    xs += [0.0, -0.0, 3.4e38, 3.3961e38, 3.3962e38, 1e-45, 2.0 ** -133, 2.0 ** -134,
           3 * 2.0 ** -135]
    xs = np.asarray(xs, dtype=np.float64)
    ours = nm.f64_to_bf16_bits(xs)
    ref = np.asarray([_exact_bf16_bits(float(v)) for v in xs], dtype=np.uint16)
    assert np.array_equal(ours, ref)


def test_f64_to_bf16_differs_from_double_rounding_on_constructed_case():
    # mid + 1 ulp(f64): f32 rounding lands on the midpoint, then ties-to-even
    # goes down; the single rounding goes up.
    mid = (129 + 0.5) * 2.0 ** -7            # between 129/128 and 130/128
    x = np.nextafter(mid, np.inf)
    single = nm.f64_to_bf16_bits(np.array([x]))[0]
    via_f32 = nm.f32_to_bf16_bits(np.array([x], dtype=np.float32))[0]
    assert single == 0x3F82 and via_f32 == 0x3F82 - 0  # 130/128 either way here
    y = np.nextafter((128 + 0.5) * 2.0 ** -7, np.inf)  # midpoint above an even code
    assert nm.f64_to_bf16_bits(np.array([y]))[0] == 0x3F81
    assert nm.f32_to_bf16_bits(np.array([y], dtype=np.float32))[0] == 0x3F80


def test_e4m3_decode_table_definition():
    t = nm.E4M3_DECODE
    assert t[0x00] == 0.0 and t[0x80] == 0.0 and math.copysign(1, t[0x80]) < 0
    assert t[0x01] == 2.0 ** -9 and t[0x07] == 7 * 2.0 ** -9
    assert t[0x08] == 2.0 ** -6 and t[0x38] == 1.0 and t[0x7E] == 448.0
    assert math.isnan(t[0x7F]) and math.isnan(t[0xFF])
    pos = t[:0x7F]
    assert np.all(np.diff(pos) > 0)
    assert np.array_equal(t[0x80:0xFF], -t[:0x7F])
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    fin = ~np.isnan(t)
    assert np.array_equal(t[fin].astype(np.float32), ref[fin])


def test_e4m3_golden_points():
    rows = [l.split() for l in open(f"{GOLDEN}/e4m3_points.txt") if l.strip() and not l.startswith("#")]
    for code, value in rows:
        assert nm.E4M3_DECODE[int(code, 16)] == float(Fraction(value))
        assert nm.e4m3_encode(np.array([float(Fraction(value))], np.float32))[0] == int(code, 16)


def test_e4m3_encode_matches_torch_in_range():
    t = nm.E4M3_DECODE[:0x7F]
    mids = (t[:-1] + t[1:]) / 2
    pts = np.concatenate([t, mids, np.linspace(0, 464, 200001)]).astype(np.float32)
    near = np.concatenate([np.nextafter(pts, np.float32(0)), np.nextafter(pts, np.float32(1e9))])
    rng = np.random.default_rng(7)
    rnd = (rng.random(200000) * np.exp2(rng.integers(-14, 9, 200000))).astype(np.float32)
    x = np.concatenate([pts, near, rnd, [464.0]]).astype(np.float32)
    x = x[np.abs(x) <= 464]
    x = np.concatenate([x, -x])
    ours = nm.e4m3_encode(x)
    ref = torch.from_numpy(x.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_saturates_and_roundtrips():
    big = np.array([464.0001, 480, 1e4, 3.4e38, np.inf], dtype=np.float32)
    assert np.all(nm.e4m3_encode(big) == 0x7E)
    assert np.all(nm.e4m3_encode(-big) == 0xFE)
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    assert np.array_equal(nm.e4m3_encode(nm.e4m3_decode(codes).astype(np.float32)), codes)


def _exact_f32(x: Fraction) -> float:
    """Reference: RNE of an exact rational onto the binary32 grid."""
    if x == 0:
        return 0.0
    ax = abs(x)
    E = math.floor(math.log2(float(ax))) if float(ax) > 0 else -200
    while Fraction(2) ** E > ax:
        E -= 1
    while Fraction(2) ** (E + 1) <= ax:
        E += 1
    E = max(E, -126)
    q = _exact_rne(ax, Fraction(2) ** (E - 23))
    if q >= Fraction(2) ** 128:
        return math.copysign(math.inf, x)
    return float(q) if x > 0 else -float(q)


def _fma_cases():
    rng = np.random.default_rng(31)
    n = 4000
    a = (rng.standard_normal(n) * np.exp2(rng.integers(-30, 30, n))).astype(np.float32)
    b = (rng.standard_normal(n) * np.exp2(rng.integers(-30, 30, n))).astype(np.float32)
    # c near -a*b (cancellation) for a third, far smaller / larger for the rest
    c = (rng.standard_normal(n) * np.exp2(rng.integers(-60, 30, n))).astype(np.float32)
    third = n // 3
    c[:third] = (-(a[:third].astype(np.float64) * b[:third]) * (1 + rng.standard_normal(third) * 1e-6)
                 ).astype(np.float32)
    # the attention exponent: integer score * FP32 multiplier + FP32 offset
    S = rng.integers(-2_000_000, 2_000_000, 2000).astype(np.float32)
    cm = (rng.uniform(1e-5, 1e-3, 2000)).astype(np.float32)
    e = (-(S.astype(np.float64) * cm) + rng.uniform(-30, 9, 2000)).astype(np.float32)
    # constructed: a*b exactly on a binary32 midpoint, c a tiny nudge either way
    mid_a = np.float32(3.0)
    mid_b = np.float32(1 + 2.0 ** -23)               # 3 * (1 + 2^-23): a binary32 midpoint
    tiny = [2.0 ** -80, -(2.0 ** -80), 2.0 ** -60, -(2.0 ** -60), 0.0]
    ca = np.full(len(tiny), mid_a, np.float32)
    cb = np.full(len(tiny), mid_b, np.float32)
    cc = np.asarray(tiny, np.float32)
    A = np.concatenate([a, S, ca, -ca])
    Bv = np.concatenate([b, cm, cb, cb])
    C = np.concatenate([c, e, cc, cc])
    return A, Bv, C


def test_fma32_matches_exact_rational_rounding():
    A, Bv, C = _fma_cases()
    got = nm.fma32(A, Bv, C)
    ref = np.asarray([_exact_f32(Fraction(float(x)) * Fraction(float(y)) + Fraction(float(z)))
                      for x, y, z in zip(A, Bv, C)], dtype=np.float32)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_fma32_single_rounding_differs_from_separate_steps():
    # 3 * (1 + 2^-23) = 3 + 2^-22 + 2^-23 is a binary32 midpoint; a nudge of
    # -2^-80 makes the exact sum round down, which a product rounded first
    # (ties to even: up) and a float64 sum rounded later (also on the midpoint)
    # both get wrong.
    a, b, c = np.float32(3.0), np.float32(1 + 2.0 ** -23), np.float32(-(2.0 ** -80))
    fused = nm.fma32(a, b, c)
    assert float(fused) == 3.0 + 2.0 ** -22
    assert float(nm.rn32(nm.rn32(np.float64(a) * np.float64(b)) + np.float64(c))) == 3.0 + 2.0 ** -21
    assert float(nm.rn32(np.float64(a) * np.float64(b) + np.float64(c))) == 3.0 + 2.0 ** -21
