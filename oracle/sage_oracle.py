"""CPU oracle for SageAttention2-style quantized attention (K/V smoothing, INT8 QK,
FP8 PV, FP32 online softmax) on BF16 [B, N, H, D] ("NHD") tensors.

TEST INFRASTRUCTURE ONLY.  Plain, slow and meant to be read against the method
step by step.  Only the tests, the package smoke check and the benchmark's
CPU-baseline leg may import it.  It shares no code with the CUDA library and
imports nothing from it.

Sources (page, section):
* "FLUX.3 Action RTX 5090 report", 02 ENGINEERING, card 03 (SageAttention2):
  INT8 QK, FP8 PV, FP32 accumulation, K smooth and V smooth kept, NHD layout.
* same page, last-round card A: K centring (token mean subtracted) fused with
  the INT8 quantization, keeping the original BF16 rounding of the centred K;
  Q uses the same scale and INT8 rule.
* same page, card C: V mean / scale / quant with V smoothing, V written in a
  transposed, padded layout.
* "MiniMax H3 on DGX Spark", 01 Precision map: Sage2++ = QK INT8 / PV FP8.
* "为什么A10也能跑得动FLUX.1", 1.1: E4M3 = 4 exponent + 3 mantissa bits.

The pages print no formula, block size or rounding rule.  The contract below
(block of 64 tokens for Q/K scales, per-channel V scales, 128-key tiles, the
rounding steps) is the plain reading stated with each function.  Every
floating-point step that the GPU does in FP32 is rounded to FP32 here
(``rn32``); exact integer dot products are formed in float64, which is exact
for |sum| < 2**53.

Parity status: pinned by tests/test_oracle_sage.py and
tests/test_oracle_granularity.py (quantizers by brute force and invariants at
every scale granularity: 64-token blocks, per token, segment-local blocks; the attention tile loop by running it with quantization off
against brute-force FP64 softmax attention; smoothing by the softmax shift
invariance; closed forms for degenerate inputs; the softmax exp2 against
numpy's exp2 within its stated error bound and exactly at integers; the fused
multiply-add against exact rational rounding; the exponent formed on biased
scores against exact rationals and, with the score bias, by brute-force
softmax; the contract's softmax against a plain reading of it, attn_fwd_plain,
within a bound derived from the E4M3 step of P).  With the exp2 and the FMA
fixed by the contract, the E4M3 codes of P are reproducible; attention parity
keeps a tolerance for the tensor core's FP32 summation order and the order of
the row-sum additions.
"""
from __future__ import annotations

import math

import numpy as np

from .numerics import (bf16_bits_to_f32, e4m3_decode, e4m3_encode,
                       f32_to_bf16_bits, f64_to_bf16_bits, fma32, rn32,
                       round_f32_to_bf16)

QK_BLOCK = 64        # tokens per INT8 scale block of Q and K
TILE = 128           # query rows per tile and keys per KV tile
SUM_BLOCK = 64       # tokens per first-level FP64 partial sum
SUM_LANES = 32       # interleaved second-level partial sums
INT8_MAX = 127.0
E4M3_MAX = 448.0
LOG2E = 1.4426950408889634
LOG2_P_UNIT = np.float32(math.log2(E4M3_MAX))   # RN32(log2 448), the P scale in the exponent
S_BIAS = np.float32(12582912.0)  # 1.5 * 2^23: integer scores are carried as the binary32 S + S_BIAS


def npad(n: int) -> int:
    """Padded token count: N rounded up to a whole 128-row tile."""
    return ((n + TILE - 1) // TILE) * TILE


# ----------------------------------------------------------------------------
# A1 / A4: column sums over tokens in a fixed FP64 order
# ----------------------------------------------------------------------------
def column_sum_f64(x: np.ndarray) -> np.ndarray:
    """Sum x[b, n, c] over n in FP64, in the contract's fixed order.

    The pages only say "subtract the mean"; to make the means (and so every
    code) reproducible the order of the FP64 additions is fixed:
      1. 64-token blocks: s_c = ((0 + x_{64c}) + x_{64c+1}) + ... in token
         order, over the block's tokens that exist (the last may be short);
      2. 32 interleaved lanes: u_g = ((0 + s_g) + s_{g+32}) + s_{g+64} + ...;
      3. butterfly over the lanes: for o in 16, 8, 4, 2, 1:
         u_g <- u_g + u_{g xor o}; the column sum is u_0.
    Input x: float32 or float64 [B, N, C]; returns float64 [B, C].
    """
    x = np.asarray(x)
    B, N, C = x.shape
    nb = (N + SUM_BLOCK - 1) // SUM_BLOCK
    partial = np.zeros((B, nb, C), dtype=np.float64)
    for c in range(nb):
        s = np.zeros((B, C), dtype=np.float64)
        for n in range(c * SUM_BLOCK, min(N, (c + 1) * SUM_BLOCK)):
            s = s + x[:, n, :].astype(np.float64)
        partial[:, c] = s
    lanes = np.zeros((B, SUM_LANES, C), dtype=np.float64)
    for g in range(SUM_LANES):
        u = np.zeros((B, C), dtype=np.float64)
        for c in range(g, nb, SUM_LANES):
            u = u + partial[:, c]
        lanes[:, g] = u
    idx = np.arange(SUM_LANES)
    o = SUM_LANES // 2
    while o >= 1:
        lanes = lanes + lanes[:, idx ^ o]
        o //= 2
    return lanes[:, 0]


# ----------------------------------------------------------------------------
# A2: INT8 block quantization (Q as is, K after centring)
# ----------------------------------------------------------------------------
GRANULARITIES = ("block64", "token", "segment64")


def scale_groups(N: int, gran: str = "block64", cu_seqlens=None) -> np.ndarray:
    """First token of every INT8 scale group on the padded token axis [0, Npad).

    Groups are runs of consecutive tokens; every group spans all D channels.
      block64    64-token blocks on one grid over the whole sequence (the
                 configurations' "Q/K INT8 blocks 64 tokens");
      token      one group per token (the tcgen05 counterpart of the pages'
                 per-thread granularity, which gives each GPU thread its own
                 scale: here one thread owns one query row);
      segment64  64-token blocks restarting at every segment start of a packed
                 joint sequence (cu_seqlens), so that no block mixes two streams;
                 the last block of a segment may be short.
    Padded tokens [N, Npad) hold zeros; in segment64 they form blocks of their
    own, on the 64-token grid that continues from N.
    """
    Np = npad(N)
    if gran == "block64":
        return np.arange(0, Np, QK_BLOCK)
    if gran == "token":
        return np.arange(Np)
    if gran == "segment64":
        cu = [0, N] if cu_seqlens is None else [int(c) for c in cu_seqlens]
        starts = []
        for a, e in zip(cu[:-1], cu[1:]):
            starts.extend(range(a, e, QK_BLOCK))
        starts.extend(range(N, Np, QK_BLOCK))
        return np.asarray(starts, dtype=np.int64)
    raise ValueError(f"unknown granularity {gran!r}")


def int8_group_quant(x: np.ndarray, starts: np.ndarray):
    """Quantize x[B, H, Npad, D] (float32, zero in padded rows) per scale group.

    starts: first token of each group (increasing, starts[0] == 0); group g is
    tokens [starts[g], starts[g+1]) over all D channels.  For each (b, h, group):
      amax  = max |x| over the group,
      scale = RN32(amax / 127),  inv = RN32(127 / amax),
      code  = clamp(RNE(RN32(x * inv)), -127, 127);
    amax == 0 gives scale = inv = 0 and all codes 0.
    Returns (codes int8 [B, H, Npad, D], scale float32 [B, H, n_groups]).
    """
    x = np.asarray(x, dtype=np.float32)
    B, H, Np, D = x.shape
    starts = np.asarray(starts, dtype=np.int64)
    lengths = np.diff(np.append(starts, Np))
    amax = np.maximum.reduceat(np.abs(x).max(axis=3), starts, axis=2)     # [B, H, G]
    nz = amax > 0
    safe = np.where(nz, amax, np.float32(1))
    scale = np.where(nz, safe / np.float32(INT8_MAX), np.float32(0)).astype(np.float32)
    inv = np.where(nz, np.float32(INT8_MAX) / safe, np.float32(0)).astype(np.float32)
    inv_tok = np.repeat(inv, lengths, axis=2)                              # [B, H, Npad]
    prod = (x * inv_tok[..., None]).astype(np.float32)
    codes = np.clip(np.rint(prod), -INT8_MAX, INT8_MAX).astype(np.int8)
    return codes, scale


def int8_block_quant(x: np.ndarray):
    """int8_group_quant on 64-token blocks: (codes [B, H, Npad, D], scale [B, H, Npad/64])."""
    return int8_group_quant(x, np.arange(0, x.shape[2], QK_BLOCK))


def quant_scales(x: np.ndarray, N: int, gran: str = "block64", cu_seqlens=None):
    """INT8 codes and scales of x[B, H, Npad, D] at a granularity, in the layout
    the attention call reads: block64 -> scale [B, H, Npad/64] (one per block);
    token, segment64 -> scale [B, H, Npad] (every token holds its group's scale)."""
    starts = scale_groups(N, gran, cu_seqlens)
    codes, scale = int8_group_quant(x, starts)
    if gran == "block64":
        return codes, scale
    lengths = np.diff(np.append(starts, x.shape[2]))
    return codes, np.repeat(scale, lengths, axis=2)


def token_scales(scale: np.ndarray, Np: int) -> np.ndarray:
    """The per-token view of a Q or K scale array in either layout."""
    if scale.shape[-1] == Np:
        return scale
    assert scale.shape[-1] * QK_BLOCK == Np, scale.shape
    return np.repeat(scale, QK_BLOCK, axis=-1)


def _nhd_to_bhnd_padded(x32: np.ndarray) -> np.ndarray:
    B, N, H, D = x32.shape
    out = np.zeros((B, H, npad(N), D), dtype=np.float32)
    out[:, :, :N, :] = np.transpose(x32, (0, 2, 1, 3))
    return out


def k_mean_bf16(k_bits: np.ndarray) -> np.ndarray:
    """A1: per-(b, h, d) token mean of K, FP64 sum, ONE rounding to BF16.

    mean = RN_bf16(sum / N) with the sum in the fixed order of column_sum_f64
    and the FP64 quotient rounded straight to BF16.  Returns uint16 [B, H, D].
    """
    B, N, H, D = k_bits.shape
    k32 = bf16_bits_to_f32(k_bits).reshape(B, N, H * D)
    s = column_sum_f64(k32)
    return f64_to_bf16_bits(s / np.float64(N)).reshape(B, H, D)


def quant_qk(q_bits: np.ndarray, k_bits: np.ndarray, q_gran: str = "block64",
             k_gran: str = "block64", cu_seqlens=None, normrope=None):
    """A1-A3: K smoothing and INT8 quantization of Q and K.

    q_bits, k_bits: BF16 bit patterns uint16 [B, N, H, D].
    normrope: None, or dict(q_w, k_w, eps, cos, sin): Q and K are first taken
    through RMSNorm and RoPE in BF16 (oracle.normrope.norm_rope_bf16), and
    everything below runs on the result.
    K is centred by its BF16 token mean (over all N tokens, whatever the scale
    granularity) and rounded back to BF16 before quantization:
    kc = RN_bf16(RN32(k - mean_k)).  Q is quantized raw (the pages keep only K
    and V smoothing).  q_gran / k_gran pick the scale groups (scale_groups).
    Returns dict with q_codes, q_scale, k_codes, k_scale (layouts as
    quant_scales) and k_mean (uint16 [B, H, D]).
    """
    N = q_bits.shape[1]
    if normrope is not None:
        from .normrope import norm_rope_bf16
        nr = normrope
        q_bits = norm_rope_bf16(q_bits, nr["q_w"], nr["eps"], nr["cos"], nr["sin"])
        k_bits = norm_rope_bf16(k_bits, nr["k_w"], nr["eps"], nr["cos"], nr["sin"])
    q32 = bf16_bits_to_f32(q_bits)
    k32 = bf16_bits_to_f32(k_bits)
    mean_bits = k_mean_bf16(k_bits)
    mean32 = bf16_bits_to_f32(mean_bits)                       # [B, H, D]
    kc = round_f32_to_bf16((k32 - mean32[:, None, :, :]).astype(np.float32))
    q_codes, q_scale = quant_scales(_nhd_to_bhnd_padded(q32), N, q_gran, cu_seqlens)
    k_codes, k_scale = quant_scales(_nhd_to_bhnd_padded(kc), N, k_gran, cu_seqlens)
    return dict(q_codes=q_codes, q_scale=q_scale, k_codes=k_codes,
                k_scale=k_scale, k_mean=mean_bits)


# ----------------------------------------------------------------------------
# A4 / A5: V smoothing and per-channel FP8 quantization, transposed layout
# ----------------------------------------------------------------------------
def v_stats(v_bits: np.ndarray):
    """A4: per-(b, h, d) mean, absmax of the centred V, and the FP8 scales.

    mean  = RN32(sum / N)      (sum in the order of column_sum_f64)
    amax  = max(RN32(vmax - mean), RN32(mean - vmin))  (= max |RN32(v - mean)|,
            because rounding is monotone)
    scale = RN32(amax / 448),  inv = RN32(448 / amax);  amax == 0 -> 0, 0.
    Returns float32 arrays [B, H, D]: mean, amax, scale, inv.
    """
    B, N, H, D = v_bits.shape
    v32 = bf16_bits_to_f32(v_bits).reshape(B, N, H * D)
    mean = rn32(column_sum_f64(v32) / np.float64(N))
    vmax = v32.max(axis=1)
    vmin = v32.min(axis=1)
    amax = np.maximum((vmax - mean).astype(np.float32), (mean - vmin).astype(np.float32))
    nz = amax > 0
    safe = np.where(nz, amax, np.float32(1))
    scale = np.where(nz, safe / np.float32(E4M3_MAX), np.float32(0)).astype(np.float32)
    inv = np.where(nz, np.float32(E4M3_MAX) / safe, np.float32(0)).astype(np.float32)
    shp = (B, H, D)
    return (mean.reshape(shp), amax.reshape(shp), scale.reshape(shp), inv.reshape(shp))


def quant_v(v_bits: np.ndarray):
    """A4-A5: centre V per channel and quantize to E4M3 with per-channel scales.

    vc = RN32(v - mean);  code = E4M3_RNE_satfinite(RN32(vc * inv)).
    Codes are written transposed, [B, H, D, Npad], with zero codes for the
    padded tokens N..Npad-1.
    Returns dict with v_codes_t (uint8), v_scale, v_mean (float32 [B, H, D]).
    """
    B, N, H, D = v_bits.shape
    mean, _, scale, inv = v_stats(v_bits)
    v32 = bf16_bits_to_f32(v_bits)                               # [B, N, H, D]
    vc = (v32 - mean[:, None, :, :]).astype(np.float32)
    codes = e4m3_encode((vc * inv[:, None, :, :]).astype(np.float32))
    out = np.zeros((B, H, D, npad(N)), dtype=np.uint8)
    out[:, :, :, :N] = np.transpose(codes, (0, 2, 3, 1))
    return dict(v_codes_t=out, v_scale=scale, v_mean=mean)


# ----------------------------------------------------------------------------
# A6-A10: tiled attention with FP32 online softmax
# ----------------------------------------------------------------------------
# exp2 of the FP32 softmax (reading: the pages fix FP32 for the softmax but not
# how exp2 is evaluated; this contract fixes it so that every P8 code is
# reproducible).  Cody-Waite split with round-to-nearest, then a polynomial
# with c0 = 1 fitted for minimax relative error on [-1/2, 1/2]
# (oracle/fit_exp2.py), then n added to the exponent field.  The per-key
# weights use a quadratic (1.96e-3 after binary32 evaluation, 32 times below
# the 6.25% relative step of the E4M3 codes they feed); the once-per-tile
# rescale factor, whose error would compound over tiles in the row sum, a
# quintic (2.2e-7).
EXP2_C = tuple(np.float32(v) for v in (1.0, 0.7029417753219604, 0.2398640364408493))
EXP2_C5 = tuple(np.float32(v) for v in (1.0, 0.6931465864181519, 0.24022166430950165,
                                        0.055510472506284714, 0.009674952365458012,
                                        0.0013202981790527701))
EXP2_MIN = np.float32(-126.0)
EXP2_ROUND = np.float32(12582912.0)   # 1.5 * 2^23


def exp2_contract(u, coeffs=EXP2_C) -> np.ndarray:
    """2^u as the contract evaluates it, every step a binary32 operation.

      x  = max(u, -126)
      xr = RN(x + 1.5 * 2^23)           the integer n = round(x) in the low bits (two's complement)
      nf = RN(xr - 1.5 * 2^23)          = n, exactly
      f  = RN(x - nf)                   exact, |f| <= 1/2
      p  = c_d; p = fma(p, f, c_k) for k = d - 1 .. 0 (coeffs = c_0 .. c_d)
      y  = the binary32 whose bits are bits(p) + (bits(xr) << 23) mod 2^32,
           i.e. n added to the exponent field of p: exactly p * 2^n for
           n >= -125 (p lies in [2^-1/2, 2^1/2]); at n = -126 a value below
           2^-125 that no E4M3 code or row sum can tell from 0.
    """
    x = np.maximum(np.asarray(u, dtype=np.float32), EXP2_MIN)
    xr = rn32(x.astype(np.float64) + np.float64(EXP2_ROUND))
    nf = rn32(xr.astype(np.float64) - np.float64(EXP2_ROUND))
    f = rn32(x.astype(np.float64) - nf.astype(np.float64))
    p = np.full(f.shape, coeffs[-1], dtype=np.float32)
    for ck in coeffs[-2::-1]:
        p = fma32(p, f, ck)
    bits = p.view(np.uint32) + (xr.view(np.uint32) << np.uint32(23))   # uint32 arithmetic wraps
    return bits.astype(np.uint32).view(np.float32)


def _exp2_alpha(x):
    return exp2_contract(x, EXP2_C5)


def _identity(x):
    return np.asarray(x, dtype=np.float64)


def _attend_rows(S, col_mult, Vt, out_mult, out_add, n_keys, rn, fma, exp2, exp2_alpha, quant_p,
                 log2_p_unit, two_pass=False, s_bias=0.0, p_codes=None):
    """Online-softmax attention over 128-key tiles for one (b, h).

    S         [R, >= n_keys] float64: exact score numerators (INT32 dot
              products, or FP64 dot products with quantization off).
    col_mult  f(j0, j1) -> [R, j1 - j0] multipliers c taking S into the exp2
              domain (dequant scales x sm_scale x log2 e).
    Vt        [D, >= n_keys] float64: the (centred, dequantized-code) values.
    out_mult  [D] per-channel output factor (the V scale); out_add [D] the V
              mean added back.
    rn        rounding applied after every step (rn32, or identity in FP64).
    fma       fused multiply-add with one rounding (fma32, or exact in FP64).
    exp2      the exp2 of the per-key weights (exp2_contract, or np.exp2 in FP64);
    exp2_alpha  the exp2 of the rescale factor (exp2_contract with the quintic).
    quant_p   P quantizer (E4M3 round trip, or identity).
    log2_p_unit  log2 of the P scale folded into the exponent: RN32(log2 448)
              with quantization on, 0 with it off.
    s_bias    the bias B the scores are carried on (S_BIAS with quantization
              on: the integer S as the binary32 S + B, exact for |S| < 2^22;
              0 with it off).

    Per tile j (keys j0..j1-1, those >= n_keys excluded):
      t     = rn(S * c)                          scores in the exp2 domain
      m_new = max(m, max_k t)                    running row max
      alpha = exp2_alpha(rn(m - m_new))          (0 on the first tile, m = -inf;
                                                 exactly 1 while m is unchanged)
      e     = rn(log2_p_unit - m_new)
      e'    = fma(-B, c, e)                      the exponent offset for biased scores
      y     = exp2(fma(S + B, c, e'))            = P~ * 448, P~ = exp2(t - m_new)
                                                 up to e's rounding
      l     = rn(rn(l * alpha) + rn(sum_k y))    row sum of the unquantized y
      P8    = quant_p(y)                         E4M3 code of y (<= 448)
      acc   = rn(rn(acc * alpha) + rn(P8 @ V))   product sum exact, then rounded
    Epilogue: o = fma(rn(acc * out_mult), rn(1 / l), out_add); the P scale
    cancels between acc and l.
    With B = 0, e' = e and y = exp2(fma(S, c, e)); with B != 0 the single
    rounding of e' shifts every exponent of a (row, c) pair by the same
    amount, at most half an ulp of B * c (below 1.5 c, under two units of the
    integer score).
    two_pass: m is the final row max from the start (alpha = 1 throughout).
    p_codes: optional uint8 array [R, >= n_keys] that receives the E4M3 code
    of every y (the code P8 stands for), key by key; the arithmetic is the same
    with or without it.
    Returns (o [R, D], m [R], l [R]).
    """
    R = S.shape[0]
    D = Vt.shape[0]
    nkv = (n_keys + TILE - 1) // TILE
    m = np.full(R, -np.inf)
    if two_pass:
        for j in range(nkv):
            j0, j1 = j * TILE, min(n_keys, (j + 1) * TILE)
            t = rn(S[:, j0:j1] * col_mult(j0, j1))
            m = np.maximum(m, t.max(axis=1))
    l = np.zeros(R)
    acc = np.zeros((R, D))
    for j in range(nkv):
        j0, j1 = j * TILE, min(n_keys, (j + 1) * TILE)
        c = col_mult(j0, j1)
        t = rn(S[:, j0:j1] * c)
        tmax = t.max(axis=1)
        m_new = m if two_pass else np.maximum(m, tmax)
        with np.errstate(invalid="ignore"):
            alpha = np.where(np.isneginf(m), 0.0, np.asarray(exp2_alpha(rn(m - m_new)), dtype=np.float64))
        if two_pass:
            alpha = np.ones(R)
        e = rn(log2_p_unit - m_new)
        c_full = np.broadcast_to(c, S[:, j0:j1].shape)
        e_off = np.asarray(fma(np.float64(-s_bias), c_full, e[:, None]), dtype=np.float64)
        y = np.asarray(exp2(fma(S[:, j0:j1] + np.float64(s_bias), c_full, e_off)), dtype=np.float64)
        l = rn(rn(l * alpha) + rn(y.sum(axis=1)))
        p8 = quant_p(y)
        if p_codes is not None:
            p_codes[:, j0:j1] = e4m3_encode(y.astype(np.float32))
        acc = rn(rn(acc * alpha[:, None]) + rn(p8 @ Vt[:, j0:j1].T))
        m = m_new
    o = np.asarray(fma(rn(acc * out_mult[None, :]), rn(1.0 / l)[:, None], out_add[None, :]),
                   dtype=np.float64)
    return o, m, l


def _fma_exact(a, b, c):
    return np.asarray(a, np.float64) * b + c


def _e4m3_round_trip(x):
    return e4m3_decode(e4m3_encode(np.asarray(x, dtype=np.float32)))


def default_sm_scale(D: int) -> np.float32:
    return np.float32(1.0 / math.sqrt(D))


def exp2_scale(sm_scale) -> np.float32:
    """sm_scale * log2(e), formed in FP64 from the FP32 sm_scale, rounded once."""
    return np.float32(np.float64(np.float32(sm_scale)) * LOG2E)


def attn_fwd(q_codes, q_scale, k_codes, k_scale, v_codes_t, v_scale, v_mean, N,
             sm_scale=None, rows=None, heads=None, two_pass=False, want_lse=False,
             want_p_codes=False):
    """A6-A10 on quantized operands; the output is the FP32 attention output.

    q_codes, k_codes int8 [B, H, Npad, D]; q_scale, k_scale f32 [B, H, Npad/64]
    (one per 64-token block) or [B, H, Npad] (one per token, see quant_scales);
    v_codes_t uint8 E4M3 [B, H, D, Npad]; v_scale, v_mean f32 [B, H, D].
    Score dequant multiplier for query row i and key j, with qs[i] and ks[j]
    the scales of the groups that hold token i of Q and token j of K:
        c = RN32(RN32(qs[i] * ks[j]) * RN32(sm_scale * log2 e)),
    the P scale 448 enters the exponent as RN32(log2 448) (P8 = E4M3(y), y =
    P~ * 448 with P~ = exp2(t - m) <= 1, with the exponent formed by
    one fused multiply-add on the biased score S + S_BIAS), the row sum holds y
    and the output factor is the V scale itself.
    sm_scale None or <= 0 means 1/sqrt(D).
    rows: optional query-row indices (< N) to evaluate; heads: optional list of
    (b, h) pairs.  Returns float32 [B, R, H, D] (unevaluated heads stay 0),
    plus lse [B, H, R] (natural log of the softmax denominator) if asked, plus
    the E4M3 codes of P, uint8 [B, H, R, N] (key j of row i holds the code of
    y = P~ * 448 formed in key j's tile), if want_p_codes.
    """
    B, H, Np, D = q_codes.shape
    if sm_scale is None or sm_scale <= 0:
        sm_scale = default_sm_scale(D)
    sl2e = exp2_scale(sm_scale)
    rows = np.arange(N) if rows is None else np.asarray(rows)
    R = rows.shape[0]
    out = np.zeros((B, R, H, D), dtype=np.float32)
    lse = np.zeros((B, H, R), dtype=np.float32)
    pc = np.zeros((B, H, R, N), dtype=np.uint8) if want_p_codes else None
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    for b, h in heads:
        Qf = q_codes[b, h, rows].astype(np.float64)
        Kf = k_codes[b, h, :N].astype(np.float64)
        S = Qf @ Kf.T                                        # exact INT32 dots
        qs = token_scales(q_scale[b, h], Np)[rows]
        ks = token_scales(k_scale[b, h], Np)

        def col_mult(j0, j1, qs=qs, ks=ks):
            kk = ks[j0:j1]
            return rn32(rn32(qs[:, None].astype(np.float64) * kk[None, :]) * np.float64(sl2e))

        Vt = e4m3_decode(v_codes_t[b, h, :, :N])
        assert np.abs(S).max(initial=0) < 2.0 ** 22          # S + S_BIAS is an exact binary32
        o, m, l = _attend_rows(S, col_mult, Vt, v_scale[b, h].astype(np.float64),
                               v_mean[b, h].astype(np.float64), N, rn32, fma32, exp2_contract,
                               _exp2_alpha, _e4m3_round_trip, LOG2_P_UNIT, two_pass=two_pass,
                               s_bias=S_BIAS, p_codes=None if pc is None else pc[b, h])
        out[b, :, h, :] = o
        lse[b, h] = rn32((m + np.log2(l) - math.log2(E4M3_MAX)) * math.log(2.0))
    res = (out,) + ((lse,) if want_lse else ()) + ((pc,) if want_p_codes else ())
    return res if len(res) > 1 else out


# ----------------------------------------------------------------------------
# The plain reading of the FP32 online softmax, kept beside the contract
# ----------------------------------------------------------------------------
def _attend_rows_plain(S, col_mult, Vt, out_mult, out_add, n_keys, rn, exp2, quant_p):
    """Online softmax over 128-key tiles in its plainest FP32 reading.

    The pages fix INT8 QK, FP8 PV, FP32 accumulation and an FP32 online
    softmax ("FLUX.3 Action RTX 5090 report", 02 ENGINEERING, card 03;
    "MiniMax H3 on DGX Spark", 01 Precision map) and nothing finer.  This
    variant takes every step as written there, with no choice made for speed:
    exp2 evaluated in FP64 and rounded once, no score bias, the running max
    exactly the largest score so far, P~ in [0, 1] scaled by 448 only for its
    E4M3 code, and l summed from the unquantized P~.

    S, col_mult, Vt, out_mult, out_add, n_keys as in _attend_rows; rn the
    rounding after every step (rn32, or identity), exp2 the exponential
    (RN32 of the FP64 exp2, or np.exp2), quant_p the P quantizer applied to
    448 * P~ (E4M3 round trip, or identity).  Per tile j:
      t     = rn(S * c)
      m_new = max(m, max_k t)
      alpha = exp2(rn(m - m_new))                (0 on the first tile)
      P~    = exp2(rn(t - m_new))                in [0, 1]
      l     = rn(rn(l * alpha) + rn(sum_k P~))
      acc   = rn(rn(acc * alpha) + rn(quant_p(rn(448 * P~)) @ V))
    Epilogue: o = rn(acc * out_mult / (448 * l) + out_add), in FP64 then
    rounded once.  Returns (o [R, D], m [R], l [R]).
    """
    R = S.shape[0]
    D = Vt.shape[0]
    nkv = (n_keys + TILE - 1) // TILE
    m = np.full(R, -np.inf)
    l = np.zeros(R)
    acc = np.zeros((R, D))
    for j in range(nkv):
        j0, j1 = j * TILE, min(n_keys, (j + 1) * TILE)
        t = rn(S[:, j0:j1] * col_mult(j0, j1))
        m_new = np.maximum(m, t.max(axis=1))
        with np.errstate(invalid="ignore"):
            alpha = np.where(np.isneginf(m), 0.0, np.asarray(exp2(rn(m - m_new)), dtype=np.float64))
        p = np.asarray(exp2(rn(t - m_new[:, None])), dtype=np.float64)
        l = rn(rn(l * alpha) + rn(p.sum(axis=1)))
        p8 = np.asarray(quant_p(rn(np.float64(E4M3_MAX) * p)), dtype=np.float64)
        acc = rn(rn(acc * alpha[:, None]) + rn(p8 @ Vt[:, j0:j1].T))
        m = m_new
    o = rn(acc * out_mult[None, :] / (np.float64(E4M3_MAX) * l)[:, None] + out_add[None, :])
    return np.asarray(o, dtype=np.float64), m, l


def _exp2_rn32(x):
    """exp2 in FP64, rounded once to binary32."""
    return rn32(np.exp2(np.asarray(x, dtype=np.float64)))


def attn_fwd_plain(q_codes, q_scale, k_codes, k_scale, v_codes_t, v_scale, v_mean, N,
                   sm_scale=None, rows=None, heads=None, quantize_p=True):
    """A6-A10 on the same quantized operands as attn_fwd, with the softmax in
    its plain reading (_attend_rows_plain): the yardstick that the contract's
    exponent (fixed quadratic exp2, biased score) is bounded against.  The
    score multiplier c, the E4M3 codes of V and the V-mean add-back are
    attn_fwd's.  quantize_p=False keeps 448 * P~ unquantized in the PV product
    (its distance from the quantized result is the plain reading's own P
    quantization error).  Returns float32 [B, R, H, D]."""
    B, H, Np, D = q_codes.shape
    if sm_scale is None or sm_scale <= 0:
        sm_scale = default_sm_scale(D)
    sl2e = exp2_scale(sm_scale)
    rows = np.arange(N) if rows is None else np.asarray(rows)
    out = np.zeros((B, rows.shape[0], H, D), dtype=np.float32)
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    for b, h in heads:
        S = q_codes[b, h, rows].astype(np.float64) @ k_codes[b, h, :N].astype(np.float64).T
        qs = token_scales(q_scale[b, h], Np)[rows]
        ks = token_scales(k_scale[b, h], Np)

        def col_mult(j0, j1, qs=qs, ks=ks):
            return rn32(rn32(qs[:, None].astype(np.float64) * ks[None, j0:j1]) * np.float64(sl2e))

        o, _, _ = _attend_rows_plain(S, col_mult, e4m3_decode(v_codes_t[b, h, :, :N]),
                                     v_scale[b, h].astype(np.float64), v_mean[b, h].astype(np.float64), N,
                                     rn32, _exp2_rn32, _e4m3_round_trip if quantize_p else _identity)
        out[b, :, h, :] = o
    return out


def attn_plain_unquantized(q, k, v, N, sm_scale=None, rows=None, heads=None):
    """_attend_rows_plain with quantization and rounding OFF, all in FP64 (no
    smoothing): pins the plain tile loop against brute-force softmax
    attention.  q, k, v float64 [B, N, H, D]; returns float64 [B, R, H, D]."""
    B, _, H, D = q.shape
    if sm_scale is None or sm_scale <= 0:
        sm_scale = 1.0 / math.sqrt(D)
    c = sm_scale * LOG2E
    rows = np.arange(N) if rows is None else np.asarray(rows)
    out = np.zeros((B, rows.shape[0], H, D))
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    for b, h in heads:
        S = q[b, rows, h, :] @ k[b, :N, h, :].T
        o, _, _ = _attend_rows_plain(S, lambda j0, j1: c, v[b, :N, h, :].T, np.ones(D), np.zeros(D), N,
                                     _identity, np.exp2, _identity)
        out[b, :, h, :] = o
    return out


def attn_unquantized(q, k, v, N, sm_scale=None, rows=None, smooth_k=True,
                     smooth_v=True, heads=None, s_bias=0.0):
    """The same tile loop with quantization OFF, all in FP64.

    q, k, v: float64 [B, N, H, D].  Scores are exact FP64 dot products, the
    multiplier is sm_scale * log2 e, P is not quantized (p_unit 1), V is
    centred by its FP64 mean (smooth_v) and K by its FP64 mean (smooth_k).
    s_bias: the score bias of the quantized loop, which must cancel.  Used to pin the tile loop, the rescaling, the
    biased exponent and the smoothing algebra against brute-force softmax
    attention.  Returns float64 [B, R, H, D].
    """
    B, _, H, D = q.shape
    if sm_scale is None or sm_scale <= 0:
        sm_scale = 1.0 / math.sqrt(D)
    c = sm_scale * LOG2E
    rows = np.arange(N) if rows is None else np.asarray(rows)
    out = np.zeros((B, rows.shape[0], H, D))
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    for b, h in heads:
        Q = q[b, rows, h, :]
        K = k[b, :N, h, :]
        if smooth_k:
            K = K - K.mean(axis=0)
        V = v[b, :N, h, :]
        mean = V.mean(axis=0) if smooth_v else np.zeros(D)
        S = Q @ K.T
        o, _, _ = _attend_rows(S, lambda j0, j1: c, (V - mean).T, np.ones(D), mean,
                               N, _identity, _fma_exact, np.exp2, np.exp2, _identity, 0.0,
                               s_bias=s_bias)
        out[b, :, h, :] = o
    return out


def attn_exact_fp64(q, k, v, N, sm_scale=None, rows=None, heads=None):
    """Plain softmax(Q K^T * sm_scale) V in FP64 on the given values, no tiling.

    q, k, v: float64 [B, N, H, D].  Returns float64 [B, R, H, D].
    """
    B, _, H, D = q.shape
    if sm_scale is None or sm_scale <= 0:
        sm_scale = 1.0 / math.sqrt(D)
    rows = np.arange(N) if rows is None else np.asarray(rows)
    out = np.zeros((B, rows.shape[0], H, D))
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    for b, h in heads:
        s = (q[b, rows, h, :] @ k[b, :N, h, :].T) * sm_scale
        s = s - s.max(axis=1, keepdims=True)
        e = np.exp(s)
        out[b, :, h, :] = (e / e.sum(axis=1, keepdims=True)) @ v[b, :N, h, :]
    return out


def sage_pipeline(q_bits, k_bits, v_bits, sm_scale=None, rows=None, heads=None,
                  two_pass=False, q_gran="block64", k_gran="block64", cu_seqlens=None, plain=False):
    """Whole path A1-A10 from BF16 inputs: returns (fp32 output, intermediates).
    plain: the softmax in its plain reading (attn_fwd_plain) instead of the contract."""
    N = q_bits.shape[1]
    qk = quant_qk(q_bits, k_bits, q_gran, k_gran, cu_seqlens)
    vv = quant_v(v_bits)
    if plain:
        o = attn_fwd_plain(qk["q_codes"], qk["q_scale"], qk["k_codes"], qk["k_scale"], vv["v_codes_t"],
                           vv["v_scale"], vv["v_mean"], N, sm_scale=sm_scale, rows=rows, heads=heads)
        return o, dict(qk, **vv)
    o = attn_fwd(qk["q_codes"], qk["q_scale"], qk["k_codes"], qk["k_scale"],
                 vv["v_codes_t"], vv["v_scale"], vv["v_mean"], N, sm_scale=sm_scale,
                 rows=rows, heads=heads, two_pass=two_pass)
    return o, dict(qk, **vv)


def bf16_output(o32: np.ndarray) -> np.ndarray:
    """The BF16 output is the RNE rounding of the FP32 output (bit patterns)."""
    return f32_to_bf16_bits(o32)
