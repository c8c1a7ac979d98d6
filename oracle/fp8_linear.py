"""CPU oracle of the row-wise FP8 projection: per-token FP8 activations times
per-output-row FP8 weights, FP32 accumulation, both scales in the epilogue.

TEST INFRASTRUCTURE ONLY (part of the CPU oracle).  Only the tests, the
package smoke check and the benchmark's CPU-baseline leg may import it.  It
shares no code with the CUDA library.

Sources (page, section):
* "FLUX.3 Action on RTX 5090" report, 02 ENGINEERING, card 02: the selected
  projections run in E4M3 with one scale per output row (the Q/K projections
  stay BF16).
* "FLUX 3 Action" (SGLang cookbook), serving notes: the FP8r packages load
  native E4M3 weights (one scale per output row) and run a scaled matrix
  product with per-token activation scales.

The pages give no rounding rule.  The reading restated here, for X [M, K] and
W [N, K] (BF16):
  per row r of X (and, offline, of W): amax = max |x|, scale = RN(amax / 448),
  inv = RN(448 / amax), code = E4M3_RNE_satfinite(RN(x * inv)); amax == 0 gives
  scale 0 and zero codes (the rule of the V quantization, applied per row);
  acc[m, n] = RN32(sum_k xq[m,k] * wq[n,k])   (the exact sum, rounded once),
  y[m, n] = RN32(RN32(acc[m, n] * sx[m]) * sw[n]);  the BF16 output is RN_bf16(y).
Every E4M3 value is an integer multiple of 2^-9 and at most 448 = 229376 * 2^-9,
so a product is an integer below 2^36 in units of 2^-18: acc is summed exactly
in int64 (any K below 2^27) and is exactly a float64 for K <= 2^17, then
rounded once.  The GPU accumulates in FP32 on the tensor cores; the parity
tests bound the difference.

Parity status: pinned by tests/test_oracle_fp8_linear.py (the quantizer by
its error bound and extreme codes, the product against float64 matrix
products and closed forms).
"""
from __future__ import annotations

import numpy as np

from .numerics import bf16_bits_to_f32, e4m3_decode, e4m3_encode, f32_to_bf16_bits, rn32

E4M3_MAX = 448.0


def fp8_quant_rows(x_bits: np.ndarray):
    """Per-row E4M3 quantization of BF16 bits [R, K]: (codes uint8 [R, K], scale f32 [R])."""
    x = bf16_bits_to_f32(x_bits)
    amax = np.abs(x).max(axis=1)
    nz = amax > 0
    safe = np.where(nz, amax, np.float32(1))
    scale = np.where(nz, safe / np.float32(E4M3_MAX), np.float32(0)).astype(np.float32)
    inv = np.where(nz, np.float32(E4M3_MAX) / safe, np.float32(0)).astype(np.float32)
    codes = e4m3_encode((x * inv[:, None]).astype(np.float32))
    return codes, scale


def _units(codes: np.ndarray) -> np.ndarray:
    """E4M3 codes as exact integers in units of 2^-9."""
    return np.rint(e4m3_decode(codes).astype(np.float64) * 512.0).astype(np.int64)


def fp8_accumulate(xq: np.ndarray, wq: np.ndarray) -> np.ndarray:
    """Exact acc[m, n] = sum_k dec(xq[m, k]) * dec(wq[n, k]) as float64 (exact).

    In units of 2^-18 every product is an integer below 2^36; for K <= 2^17
    every partial sum stays below 2^53, so a float64 matrix product of the
    integer units is exact in any summation order; beyond that, int64."""
    a = _units(xq)
    b = _units(wq)
    if xq.shape[1] <= 1 << 17:
        acc = a.astype(np.float64) @ b.T.astype(np.float64)
    else:
        acc = (a @ b.T).astype(np.float64)
    return acc * 2.0 ** -18


def fp8_linear(xq, sx, wq, sw) -> np.ndarray:
    """y[m, n] = RN32(RN32(acc * sx[m]) * sw[n]) with acc the exact sum rounded
    once to binary32 (float32 [M, N]; products of binary32 values are exact in
    float64, so each RN32 below is a single rounding)."""
    acc = rn32(fp8_accumulate(xq, wq)).astype(np.float64)
    t = rn32(acc * np.asarray(sx, np.float32).astype(np.float64)[:, None])
    return rn32(t.astype(np.float64) * np.asarray(sw, np.float32).astype(np.float64)[None, :])


def fp8_linear_bf16(x_bits, wq, sw) -> np.ndarray:
    """The whole projection from BF16 activations: quantize X per token, multiply,
    scale, round to BF16.  Returns BF16 bits [M, N]."""
    xq, sx = fp8_quant_rows(x_bits)
    return f32_to_bf16_bits(fp8_linear(xq, sx, wq, sw))
