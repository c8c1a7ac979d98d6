"""Number formats used by the quantized-attention contract, written out on the CPU.

TEST INFRASTRUCTURE ONLY.  This module belongs to the CPU oracle.  Only the test
suite, the package smoke check and the benchmark's CPU-baseline leg may import
it; the CUDA library never does, and it imports nothing from the CUDA side.

Formats (each function states the rule it implements):

* BF16: 1 sign, 8 exponent, 7 mantissa bits; the upper half of an IEEE binary32.
  The BF16 inputs of the attention calls are held as raw uint16 bit patterns.
* E4M3 (the OCP "FP8 E4M3FN" format): 1 sign, 4 exponent, 3 mantissa bits,
  exponent bias 7, no infinities, S.1111.111 is NaN, largest finite 448.
  The 4+3 split is the one the FLUX.1 FP8 article states ("为什么A10也能跑得动
  FLUX.1", section 1.1); the bias, the NaN code and the 448 maximum are the
  format's published definition.

Rounding is always round-to-nearest, ties-to-even (RNE), done by scaling the
value onto the target's unit in the last place and calling ``np.rint``, which
is RNE and exact for the magnitudes involved.  Parity status: pinned (tests in
tests/test_oracle_numerics.py compare every function with torch's casts or with
exact rational arithmetic).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


# ----------------------------------------------------------------------------
# BF16
# ----------------------------------------------------------------------------
def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """BF16 bit patterns (uint16) -> float32 values (exact widening)."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> BF16 bits, round to nearest even (finite inputs; NaN kept NaN).

    Rule: keep the upper 16 bits of the binary32 pattern after adding half an
    ulp of BF16 (0x7FFF) plus the lowest kept bit, which breaks ties to even.
    Overflow past the largest BF16 carries into the exponent and yields inf.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)
    nan = np.isnan(np.asarray(x, dtype=np.float32))
    if nan.any():
        r = np.where(nan, (u >> np.uint64(16)).astype(np.uint16) | np.uint16(0x0040), r)
    return r


def round_f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> float32 value of its BF16 rounding (RNE)."""
    return bf16_bits_to_f32(f32_to_bf16_bits(x))


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float64 -> BF16 bits with ONE rounding (RNE), not via binary32.

    The BF16 unit in the last place of a value with binary exponent E
    (2**E <= |x| < 2**(E+1)) is 2**(E-7); below the smallest normal 2**-126
    it is fixed at 2**-133 (subnormals).  |x| is scaled onto that unit, rounded
    with rint (RNE, exact: the scaled value is below 2**9) and scaled back.  The
    result is exactly representable in BF16 (or overflows to inf), so reading
    its binary32 pattern and keeping the upper half gives the code.
    """
    x = np.asarray(x, dtype=np.float64)
    ax = np.abs(x)
    _, e = np.frexp(ax)                 # ax = f * 2**e, f in [0.5, 1)
    E = e.astype(np.int64) - 1          # 2**E <= ax < 2**(E+1)
    E = np.maximum(E, -126)             # subnormal range shares one unit
    unit = np.ldexp(1.0, (E - 7).astype(np.int64))
    q = np.rint(ax / unit) * unit       # power-of-two scaling is exact
    with np.errstate(over="ignore"):
        v = np.where(np.signbit(x), -q, q).astype(np.float32)
    bits = (v.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        bits = np.where(nan, np.uint16(0x7FC0), bits)
    return bits


def f64_to_f32(x: np.ndarray) -> np.ndarray:
    """float64 -> float32 with RNE (IEEE conversion)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def fma32(a, b, c) -> np.ndarray:
    """IEEE binary32 fused multiply-add: RNE of the exact a*b + c, one rounding.

    a, b, c are float32 values (any array-like; broadcast).  The product of two
    binary32 numbers has at most 48 significant bits, so it is exact in
    float64.  The sum is taken in float64 together with its exact error
    (Knuth's TwoSum), and the float64 sum is rounded to binary32.  That double
    rounding can only go wrong when the float64 sum lies exactly on a binary32
    midpoint while the exact sum does not; then the error term's sign picks
    the neighbour the exact sum is closer to.
    """
    a64 = np.asarray(a, dtype=np.float32).astype(np.float64)
    b64 = np.asarray(b, dtype=np.float32).astype(np.float64)
    c64 = np.asarray(c, dtype=np.float32).astype(np.float64)
    p = a64 * b64                                   # exact
    s = p + c64
    bv = s - p
    err = (p - (s - bv)) + (c64 - bv)               # exact: p + c == s + err
    r = s.astype(np.float32)
    with np.errstate(invalid="ignore", over="ignore"):
        r64 = r.astype(np.float64)
        d = s - r64                                 # exact: r is a binary32 neighbour of s
        toward = np.where(d > 0, np.float32(np.inf), np.float32(-np.inf))
        nxt = np.nextafter(r, toward)
        mid = np.isfinite(r64) & (d != 0) & (2.0 * d == nxt.astype(np.float64) - r64)
        fix = mid & (np.sign(err) == np.sign(d)) & (err != 0)
    return np.where(fix, nxt, r).astype(np.float32)


# ----------------------------------------------------------------------------
# E4M3 (FP8)
# ----------------------------------------------------------------------------
def _e4m3_decode_table() -> np.ndarray:
    t = np.empty(256, dtype=np.float64)
    for code in range(256):
        s = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            t[code] = np.nan
        elif e == 0:
            t[code] = s * m * 2.0 ** -9          # subnormal: m/8 * 2**(1-7)
        else:
            t[code] = s * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return t


E4M3_DECODE = _e4m3_decode_table()


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """E4M3 codes (uint8) -> float64 values (exact)."""
    return E4M3_DECODE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """float32 -> E4M3 codes (uint8): RNE, then saturate to +-448 (satfinite).

    The E4M3 unit in the last place for 2**E <= |x| < 2**(E+1) is 2**(E-3);
    below the smallest normal 2**-6 it is 2**-9.  |x| is scaled onto that unit
    and rounded with rint (RNE); a carry to the next binade stays exact.  The
    rounded magnitude is then clamped to 448, which is what rounding with an
    unbounded exponent followed by saturation to the largest finite value
    gives.  NaN maps to the NaN code 0x7F (sign kept).
    """
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    ax = np.abs(x)
    _, e = np.frexp(ax)
    E = np.maximum(e.astype(np.int64) - 1, -6)
    unit = np.ldexp(1.0, (E - 3).astype(np.int64))
    q = np.minimum(np.rint(ax / unit) * unit, E4M3_MAX)
    # q is now an exact E4M3 magnitude: rebuild its code.
    _, e2 = np.frexp(q)
    E2 = e2.astype(np.int64) - 1
    normal = q >= 2.0 ** -6
    exp_field = np.where(normal, E2 + 7, 0)
    man_field = np.where(normal,
                         np.rint((q / np.ldexp(1.0, E2) - 1.0) * 8.0),
                         np.rint(q / 2.0 ** -9))
    code = (exp_field << 3) | man_field.astype(np.int64)
    code = np.where(np.signbit(x), code | 0x80, code)
    code = np.where(np.isnan(x), np.where(np.signbit(x), 0xFF, 0x7F), code)
    return code.astype(np.uint8)


def rn32(x) -> np.ndarray:
    """Round a float64 intermediate to binary32 (RNE)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32)
