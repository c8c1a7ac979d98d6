"""CPU oracle of the step that feeds the quantized attention: RMSNorm of each Q
and K head vector followed by the rotary position embedding, in BF16 rounding.

TEST INFRASTRUCTURE ONLY (part of the CPU oracle).  Only the tests, the
package smoke check and the benchmark's CPU-baseline leg may import it.  It
shares no code with the CUDA library.

Sources (page, section):
* "FLUX 3 Action" (SGLang cookbook), 1 Model Introduction: the joint blocks use
  a 4-axis (t, h, w, l) RoPE; the serving notes: QK RMSNorm + RoPE run as one
  fused kernel at BF16 rounding level (an eager path exists beside it).
* "FLUX.3 Action on RTX 5090" report, last-round card B: the Norm / RoPE kernel
  writes BF16 in the NHD layout that the attention reads.

The pages give no formula for either step.  The reading restated here is the
eager BF16 computation of the usual QK-norm block: the mean square in FP32, the
reciprocal root, the product rounded to BF16, the learned weight applied as a
BF16 product, then the rotation of adjacent channel pairs (2i, 2i+1) in FP32,
rounded to BF16.  The order of the FP32 sum of squares is fixed (lane g of D/8
lanes sums channels 8g .. 8g+7 in order from +0; then u_g <- u_g + u_{g xor o}
for o = D/16, ..., 2, 1; the result is lane 0's), and the square root and the
division are the correctly rounded binary32 operations, so every output bit is
reproducible.  The cos / sin tables (binary32, [N, D/2], one angle per token
and channel pair) are inputs.

Parity status: pinned by tests/test_oracle_normrope.py (closed forms of the
norm and of the rotation, an FP64 restatement within BF16 rounding, the sum's
order against an exact sum, the pairing convention on a hand example).
"""
from __future__ import annotations

import numpy as np

from .numerics import bf16_bits_to_f32, f32_to_bf16_bits, rn32


def _to_bf16_f32(x32: np.ndarray) -> np.ndarray:
    """RN_bf16 of binary32 values, returned as binary32."""
    return bf16_bits_to_f32(f32_to_bf16_bits(np.asarray(x32, dtype=np.float32)))


def sum_of_squares_f32(x32: np.ndarray) -> np.ndarray:
    """Sum of x**2 over the last axis (D, a multiple of 8) in the fixed FP32 order.

    x**2 of a BF16 value is exact in binary32, so each step is one rounding:
    lane g accumulates channels 8g .. 8g+7 in order, then the lanes combine in a
    butterfly over o = L/2, ..., 1 (L = D/8 lanes), and lane 0 holds the sum.
    """
    x32 = np.asarray(x32, dtype=np.float32)
    D = x32.shape[-1]
    L = D // 8
    sq = (x32 * x32).astype(np.float32).reshape(x32.shape[:-1] + (L, 8))   # exact squares
    lanes = np.zeros(x32.shape[:-1] + (L,), dtype=np.float32)
    for i in range(8):
        lanes = (lanes + sq[..., i]).astype(np.float32)
    idx = np.arange(L)
    o = L // 2
    while o >= 1:
        lanes = (lanes + lanes[..., idx ^ o]).astype(np.float32)
        o //= 2
    return lanes[..., 0]


def rms_norm_bf16(x_bits: np.ndarray, w_bits: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis (one head vector of D channels).

    x_bits BF16 bit patterns [..., D]; w_bits BF16 [D]; eps a binary32 value.
      ms = RN32(sum_of_squares / D)        (D a power of two: exact scaling)
      r  = RN32(1 / RN32(sqrt(RN32(ms + eps))))
      y  = RN_bf16(RN32(x * r))
      z  = RN_bf16(y * w)                  (y * w is exact in binary32)
    Returns BF16 bit patterns of z.
    """
    x32 = bf16_bits_to_f32(x_bits)
    w32 = bf16_bits_to_f32(w_bits)
    D = x32.shape[-1]
    ms = (sum_of_squares_f32(x32) / np.float32(D)).astype(np.float32)
    den = np.sqrt((ms + np.float32(eps)).astype(np.float32)).astype(np.float32)
    r = (np.float32(1.0) / den).astype(np.float32)
    y = _to_bf16_f32((x32 * r[..., None]).astype(np.float32))
    z = (y * w32).astype(np.float32)
    return f32_to_bf16_bits(z)


def rope_bf16(x_bits: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotate adjacent channel pairs of x_bits [B, N, H, D] (BF16 bits).

    cos, sin: binary32 [N, D/2]; pair i of token n turns by the angle whose
    cosine and sine are cos[n, i], sin[n, i]:
      a, b = x[..., 2i], x[..., 2i+1]
      o0 = RN32(RN32(cos * a) - RN32(sin * b))
      o1 = RN32(RN32(sin * a) + RN32(cos * b))
    then both rounded to BF16.  Returns BF16 bit patterns.
    """
    x32 = bf16_bits_to_f32(x_bits)
    c = np.asarray(cos, dtype=np.float32)[None, :, None, :]
    s = np.asarray(sin, dtype=np.float32)[None, :, None, :]
    a = x32[..., 0::2]
    b = x32[..., 1::2]
    o0 = rn32(rn32(c.astype(np.float64) * a) - rn32(s.astype(np.float64) * b))
    o1 = rn32(rn32(s.astype(np.float64) * a) + rn32(c.astype(np.float64) * b))
    out = np.empty_like(x32)
    out[..., 0::2] = o0
    out[..., 1::2] = o1
    return f32_to_bf16_bits(out)


def norm_rope_bf16(x_bits: np.ndarray, w_bits: np.ndarray, eps: float, cos: np.ndarray,
                   sin: np.ndarray) -> np.ndarray:
    """RMSNorm then RoPE of x_bits [B, N, H, D]; BF16 bits in, BF16 bits out."""
    return rope_bf16(rms_norm_bf16(x_bits, w_bits, eps), cos, sin)
