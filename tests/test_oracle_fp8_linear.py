"""Pins of the oracle's row-wise FP8 projection (oracle/fp8_linear.py): the
per-row E4M3 quantizer by hand values, its error bound and extreme codes; the
exact accumulation against rational arithmetic and float64 matrix products;
the scaled product by power-of-two identities and a closed form."""
from fractions import Fraction

import numpy as np

import synth
from oracle import fp8_linear as fl
from oracle.numerics import bf16_bits_to_f32, e4m3_decode


def _bf(x):
    return synth.to_bf16_bits(np.asarray(x, dtype=np.float32))


def test_quant_rows_hand_values():
    # amax 448: scale 1, inv 1, the codes are the E4M3 encodings of the values
    x = _bf([[448.0, 224.0, 1.0, -3.5, 0.0, 17.0, -448.0, 0.01953125]])
    codes, scale = fl.fp8_quant_rows(x)
    assert scale[0] == 1.0
    assert np.array_equal(e4m3_decode(codes[0]), [448, 224, 1, -3.5, 0, 16, -448, 0.01953125])
    # an all-zero row: zero scale and codes
    c0, s0 = fl.fp8_quant_rows(_bf(np.zeros((2, 16))))
    assert not c0.any() and not s0.any()


def test_quant_rows_bound_and_extremes():
    rng = np.random.default_rng(1)
    x = _bf(rng.standard_normal((64, 256)) * np.exp(rng.standard_normal((64, 1)) * 3))
    codes, scale = fl.fp8_quant_rows(x)
    xf = bf16_bits_to_f32(x).astype(np.float64)
    dec = e4m3_decode(codes)
    assert np.all(np.abs(dec).max(axis=1) == 448.0)        # the row's absmax lands on 448
    # E4M3 spacing at |v| is at most 2^-3 |v| (normal) and 2^-9 (subnormal)
    v = np.abs(xf) / scale[:, None]
    step = np.maximum(v * 2.0 ** -3, 2.0 ** -9)
    assert np.all(np.abs(dec - xf / scale[:, None]) <= 0.5 * step * (1 + 1e-6) + 448 * 2.0 ** -23)


def test_accumulation_exact():
    rng = np.random.default_rng(2)
    xq = rng.integers(0, 256, size=(5, 24), dtype=np.uint8)
    wq = rng.integers(0, 256, size=(3, 24), dtype=np.uint8)
    xq[(xq & 0x7F) == 0x7F] = 0                            # no NaN codes
    wq[(wq & 0x7F) == 0x7F] = 0
    acc = fl.fp8_accumulate(xq, wq)
    for m in range(5):
        for n in range(3):
            exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(e4m3_decode(xq[m]), e4m3_decode(wq[n])))
            assert Fraction(acc[m, n]) == exact


def test_linear_power_of_two_identities_and_closed_form():
    rng = np.random.default_rng(3)
    M, N, K = 16, 12, 64
    x = _bf(rng.standard_normal((M, K)))
    w = _bf(rng.standard_normal((N, K)) * 0.05)
    wq, sw = fl.fp8_quant_rows(w)
    xq, sx = fl.fp8_quant_rows(x)
    y = fl.fp8_linear(xq, sx, wq, sw)
    # scaling a row of X (or of W) by 2^k scales exactly that row (column) of y by 2^k
    x2 = bf16_bits_to_f32(x).copy()
    x2[3] *= 8.0
    xq2, sx2 = fl.fp8_quant_rows(_bf(x2))
    y2 = fl.fp8_linear(xq2, sx2, wq, sw)
    assert np.array_equal(y2[3], 8.0 * y[3]) and np.array_equal(np.delete(y2, 3, 0), np.delete(y, 3, 0))
    w2 = bf16_bits_to_f32(w).copy()
    w2[5] *= 0.25
    wq2, sw2 = fl.fp8_quant_rows(_bf(w2))
    y3 = fl.fp8_linear(xq, sx, wq2, sw2)
    assert np.array_equal(y3[:, 5], 0.25 * y[:, 5])
    # against the float64 product of the dequantized matrices (exact sums, one rounding each)
    ref = (e4m3_decode(xq) * sx[:, None].astype(np.float64)) @ (e4m3_decode(wq) * sw[:, None].astype(np.float64)).T
    assert np.allclose(y, ref, rtol=3 * 2.0 ** -24, atol=0)
    # W = identity: y is the dequantized X (within E4M3 rounding of X)
    eye = fl.fp8_quant_rows(_bf(np.eye(K)))
    yi = fl.fp8_linear(xq, sx, *eye)
    xf = bf16_bits_to_f32(x).astype(np.float64)
    assert np.all(np.abs(yi - xf) <= np.abs(xf) * 2.0 ** -4 + sx[:, None] * 2.0 ** -9 + 1e-7)


def test_float64_and_int64_accumulations_agree():
    rng = np.random.default_rng(5)
    xq = rng.integers(0, 256, size=(4, 4096), dtype=np.uint8)
    wq = rng.integers(0, 256, size=(6, 4096), dtype=np.uint8)
    xq[(xq & 0x7F) == 0x7F] = 0
    wq[(wq & 0x7F) == 0x7F] = 0
    a = fl._units(xq)
    b = fl._units(wq)
    assert np.array_equal(fl.fp8_accumulate(xq, wq), (a @ b.T).astype(np.float64) * 2.0 ** -18)
