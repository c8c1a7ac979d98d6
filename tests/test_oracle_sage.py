"""Pins for the oracle's method steps (CPU only).

Each test checks the oracle against something other than itself: exact sums,
brute-force rounding with rationals, the softmax shift invariance, brute-force
FP64 softmax attention, or a closed form of a degenerate input.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import synth
from oracle import numerics as nm
from oracle import sage_oracle as so


def _bf16(x):
    return synth.to_bf16_bits(np.asarray(x, dtype=np.float32))


# ---------------------------------------------------------------- column sums
@pytest.mark.parametrize("N", [1, 63, 64, 65, 500, 1100])
def test_column_sum_exact_when_no_rounding(N):
    rng = np.random.default_rng(N)
    x = rng.integers(-1000, 1000, size=(2, N, 5)).astype(np.float32)
    s = so.column_sum_f64(x)
    assert np.array_equal(s, x.astype(np.int64).sum(axis=1).astype(np.float64))


def test_column_sum_within_fp64_error_bound():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((1, 3000, 4)) * np.exp2(rng.integers(-30, 30, (1, 3000, 4)))).astype(np.float32)
    s = so.column_sum_f64(x)
    for c in range(4):
        exact = math.fsum(x[0, :, c].astype(np.float64))
        bound = 3000 * 2.0 ** -53 * np.abs(x[0, :, c]).astype(np.float64).sum()
        assert abs(s[0, c] - exact) <= bound


def test_k_mean_is_exact_quotient_rounded_once():
    rng = np.random.default_rng(11)
    B, N, H, D = 1, 300, 2, 16
    k = _bf16(rng.standard_normal((B, N, H, D)) * 3 + 1.5)
    mean = so.k_mean_bf16(k)
    kf = nm.bf16_bits_to_f32(k).astype(np.float64)
    for h in range(H):
        for d in range(D):
            s = math.fsum(kf[0, :, h, d])             # exact here: small spread
            q = Fraction(s) / N
            E = math.floor(math.log2(abs(float(q))))
            unit = Fraction(2) ** (E - 7)
            r = Fraction(round(q / unit)) * unit
            assert nm.bf16_bits_to_f32(mean[0, h, d:d + 1])[0] == float(r)


# ---------------------------------------------------------------- INT8 blocks
def test_int8_block_quant_brute_force_and_invariants():
    rng = np.random.default_rng(12)
    x = (rng.standard_normal((2, 3, 256, 32)) * rng.uniform(0.01, 50, (2, 3, 256, 1))).astype(np.float32)
    x[1, 2, 64:128] = 0.0                                # an all-zero block
    codes, scale = so.int8_block_quant(x)
    assert codes.dtype == np.int8 and scale.shape == (2, 3, 4)
    assert codes.min() >= -127 and codes.max() <= 127
    assert scale[1, 2, 1] == 0 and not codes[1, 2, 64:128].any()
    for b in range(2):
        for h in range(3):
            for blk in range(4):
                xb = x[b, h, blk * 64:(blk + 1) * 64].astype(np.float64)
                cb = codes[b, h, blk * 64:(blk + 1) * 64]
                amax = np.abs(xb).max()
                if amax == 0:
                    continue
                assert np.abs(cb).max() == 127
                assert scale[b, h, blk] == np.float32(amax / 127.0)
                # exact rational rounding except within 1e-4 of a tie
                ideal = xb * 127.0 / amax
                frac = np.abs(ideal - np.floor(ideal) - 0.5)
                ok = frac > 1e-4
                assert np.array_equal(cb[ok], np.rint(ideal[ok]).astype(np.int8))
                err = np.abs(cb.astype(np.float64) * scale[b, h, blk] - xb)
                assert np.all(err <= scale[b, h, blk] * (0.5 + 1e-5))


def test_block_index_mapping():
    x = np.ones((1, 1, 256, 8), dtype=np.float32)
    x[0, 0, 130, 3] = 1000.0                             # lives in block 2 only
    codes, scale = so.int8_block_quant(x)
    assert np.allclose(scale[0, 0], [1 / 127, 1 / 127, 1000 / 127, 1 / 127])
    assert np.all(codes[0, 0, :128] == 127) and np.all(codes[0, 0, 192:] == 127)
    assert codes[0, 0, 130, 3] == 127 and codes[0, 0, 131, 0] == 0


def test_quant_qk_k_smoothing_removes_channel_offsets():
    rng = np.random.default_rng(13)
    B, N, H, D = 1, 256, 2, 16
    vals = (2 * np.arange(-8, 8, dtype=np.float32) + 1) / 4      # +-1/4 .. +-15/4, zero mean
    base = rng.permuted(np.tile(vals, (B, H, D, N // 16)), axis=-1)
    base = np.transpose(base, (0, 3, 1, 2)).copy()      # each column: zero-mean, BF16-exact
    offs = rng.integers(-20, 20, size=(B, 1, H, D)).astype(np.float32)
    q = _bf16(rng.standard_normal((B, N, H, D)))
    a = so.quant_qk(q, _bf16(base))
    b = so.quant_qk(q, _bf16(base + offs))
    assert np.array_equal(nm.bf16_bits_to_f32(b["k_mean"]), offs[:, 0])
    assert np.array_equal(a["k_codes"], b["k_codes"]) and np.array_equal(a["k_scale"], b["k_scale"])
    assert np.array_equal(a["q_codes"], b["q_codes"])


def test_quant_qk_layout_and_padding():
    B, N, H, D = 1, 130, 3, 64
    q = np.zeros((B, N, H, D), np.float32)
    q[0, 129, 2, 5] = 2.0
    out = so.quant_qk(_bf16(q), _bf16(np.zeros_like(q)))
    qc = out["q_codes"]
    assert qc.shape == (B, H, 256, D) and out["q_scale"].shape == (B, H, 4)
    assert qc[0, 2, 129, 5] == 127 and np.count_nonzero(qc) == 1
    assert out["q_scale"][0, 2, 2] == np.float32(2 / 127) and out["q_scale"][0, 2, 3] == 0


# ---------------------------------------------------------------- V FP8
def test_quant_v_error_bound_layout_and_padding():
    rng = np.random.default_rng(14)
    B, N, H, D = 2, 200, 3, 32
    v32 = (rng.standard_normal((B, N, H, D)) * 2 + rng.standard_normal((B, 1, H, D)) * 5).astype(np.float32)
    v = _bf16(v32)
    out = so.quant_v(v)
    ct, sc, mean = out["v_codes_t"], out["v_scale"], out["v_mean"]
    assert ct.shape == (B, H, D, 256) and not ct[..., N:].any()
    vf = nm.bf16_bits_to_f32(v).astype(np.float64)
    exact_mean = vf.mean(axis=1)
    assert np.allclose(mean, exact_mean, rtol=1e-6, atol=1e-6)
    dec = nm.e4m3_decode(np.transpose(ct[..., :N], (0, 3, 1, 2)))   # [B, N, H, D]
    inv = np.float32(448) / (sc * 448).astype(np.float32)
    vc = vf - mean[:, None].astype(np.float64)
    x = vc * (448.0 / (sc.astype(np.float64) * 448.0))[:, None]
    half_ulp = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10)
    assert np.all(np.abs(dec - x) <= half_ulp * (1 + 1e-5) + 1e-4)
    assert np.all(np.abs(dec).max(axis=1) == 448.0)                 # channel max maps to 448
    recon = dec * sc[:, None] + mean[:, None]
    assert np.all(np.abs(recon - vf) <= np.abs(vc) * 2.0 ** -4 + sc[:, None] * 2.0 ** -9 + 1e-5)


def test_quant_v_single_spike_position():
    v = np.zeros((1, 130, 2, 64), np.float32)
    v[0, 77, 1, 9] = 130.0
    out = so.quant_v(_bf16(v))
    ct = out["v_codes_t"]
    nz = np.argwhere(ct == ct[0, 1, 9, 77])
    assert ct[0, 1, 9, 77] != ct[0, 1, 9, 76]
    assert out["v_mean"][0, 1, 9] == np.float32(1.0)
    assert out["v_scale"][0, 0, 0] == 0 and not ct[0, 0].any()


# ---------------------------------------------------------------- attention
def _rand_f64(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


@pytest.mark.parametrize("B,N,H,D", [(1, 1, 1, 64), (1, 100, 2, 64), (1, 128, 1, 128),
                                     (2, 300, 2, 64), (1, 1000, 1, 128)])
def test_tile_loop_quant_off_equals_brute_force(B, N, H, D):
    q = _rand_f64((B, N, H, D), 1, 1.5)
    k = _rand_f64((B, N, H, D), 2, 1.5) + _rand_f64((B, 1, H, D), 3, 4)
    v = _rand_f64((B, N, H, D), 4) + _rand_f64((B, 1, H, D), 5, 2)
    ref = so.attn_exact_fp64(q, k, v, N)
    got = so.attn_unquantized(q, k, v, N)
    assert np.abs(got - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())
    # The score bias cancels: the same loop with the quantized path's
    # B = 1.5 * 2^23 (FP64 rounding of the biased product and offset,
    # ~2^-52 * B * c, is the only difference).
    got_b = so.attn_unquantized(q, k, v, N, s_bias=float(so.S_BIAS))
    assert np.abs(got_b - ref).max() <= 1e-7 * max(1.0, np.abs(ref).max())


def test_biased_exponent_is_one_rounding_of_the_offset():
    """u = fma(S + B, c, e') with e' = fma(-B, c, e): within half an ulp of e'
    plus half an ulp of u of the exact S * c + e (rationals), for integer
    scores up to the INT8 maximum 127^2 * 128 and multipliers over 18 binades.
    The wrong-sign offset (e' = fma(+B, c, e)) is off by 2 B c."""
    rng = np.random.default_rng(31)
    n = 300
    smax = 127 * 127 * 128
    S = np.concatenate([[0, smax, -smax, 1, -1], rng.integers(-smax, smax + 1, n - 5)]).astype(np.float64)
    c = np.float32(2.0) ** rng.uniform(-20, -2, n).astype(np.float32)
    c = (c * np.float32(1) + np.float32(0) * c).astype(np.float32)
    e = rng.uniform(-40, 9, n).astype(np.float32)
    B = so.S_BIAS
    e_off = nm.fma32(-B, c, e)
    u = nm.fma32(S + np.float64(B), c, e_off)
    for i in range(n):
        exact = Fraction(int(S[i])) * Fraction(float(c[i])) + Fraction(float(e[i]))
        bound = Fraction(float(np.spacing(np.abs(e_off[i])))) / 2 + Fraction(float(np.spacing(np.abs(u[i])))) / 2
        assert abs(Fraction(float(u[i])) - exact) <= bound, i
    wrong = nm.fma32(S + np.float64(B), c, nm.fma32(B, c, e))
    assert np.all(np.abs(wrong.astype(np.float64) - u) >= 1.9 * float(B) * c.astype(np.float64))


def test_running_max_rule():
    """One row, three 128-key tiles with maxima 5, 4.5 and 10 (multiplier 1):
    the first tile sets m = 5, the second leaves it (alpha exactly 1 in the
    contract's exp2), the third raises it to 10; the output is the brute-force
    softmax."""
    rng = np.random.default_rng(32)
    n = 384
    S = rng.uniform(-4, 4, (1, n))
    S[0, 17], S[0, 200], S[0, 300] = 5.0, 4.5, 10.0
    V = rng.standard_normal((4, n))
    args = (S, lambda j0, j1: 1.0, V, np.ones(4), np.zeros(4), n, so._identity, so._fma_exact,
            np.exp2, np.exp2, so._identity, 0.0)
    o, m, _ = so._attend_rows(*args)
    assert m[0] == 10.0
    w = np.exp2(S[0] - S[0].max())
    assert np.allclose(o[0], (w / w.sum()) @ V.T, rtol=0, atol=1e-12)
    assert so._exp2_alpha(np.float32(0.0)) == np.float32(1.0)


def test_k_smoothing_is_softmax_invariant():
    B, N, H, D = 1, 333, 2, 64
    q, k, v = (_rand_f64((B, N, H, D), s) for s in (6, 7, 8))
    k = k + _rand_f64((B, 1, H, D), 9, 5)
    a = so.attn_unquantized(q, k, v, N, smooth_k=True)
    b = so.attn_unquantized(q, k, v, N, smooth_k=False)
    assert np.abs(a - b).max() <= 1e-12


def test_v_smoothing_is_undone_by_adding_mean_back():
    B, N, H, D = 1, 257, 2, 64
    q, k, v = (_rand_f64((B, N, H, D), s) for s in (10, 11, 12))
    v = v + _rand_f64((B, 1, H, D), 13, 3)
    a = so.attn_unquantized(q, k, v, N, smooth_v=True)
    b = so.attn_unquantized(q, k, v, N, smooth_v=False)
    assert np.abs(a - b).max() <= 1e-12


def _pipeline(q32, k32, v32, **kw):
    return so.sage_pipeline(_bf16(q32), _bf16(k32), _bf16(v32), **kw)


def test_closed_form_zero_q_gives_mean_of_dequantized_v():
    rng = np.random.default_rng(15)
    B, N, H, D = 1, 300, 2, 64
    v = rng.standard_normal((B, N, H, D)) + 2
    o, it = _pipeline(np.zeros((B, N, H, D)), rng.standard_normal((B, N, H, D)), v)
    dec = nm.e4m3_decode(it["v_codes_t"][..., :N]) * it["v_scale"][..., None] + it["v_mean"][..., None]
    expect = dec.mean(axis=-1)                                   # [B, H, D]
    assert np.abs(o - expect[:, None]).max() <= 1e-5


def test_closed_form_single_token_returns_v():
    rng = np.random.default_rng(16)
    B, N, H, D = 2, 1, 3, 64
    v = rng.standard_normal((B, N, H, D)) * 3
    o, it = _pipeline(rng.standard_normal((B, N, H, D)), rng.standard_normal((B, N, H, D)), v)
    vb = nm.bf16_bits_to_f32(_bf16(v))
    assert np.abs(o - vb).max() <= 1e-5                           # vc = 0 exactly: O = mean = v


def test_closed_form_dominant_key():
    rng = np.random.default_rng(17)
    B, N, H, D = 1, 256, 1, 64
    q = rng.standard_normal((B, N, H, D)) * 0.01
    k = rng.standard_normal((B, N, H, D)) * 0.01
    q[0, 5, 0] = 4.0
    k[0, 200, 0] = 4.0                                            # q5 . k200 = 16 dims * 16
    v = rng.standard_normal((B, N, H, D))
    o, it = _pipeline(q, k, v)
    dec_all = nm.e4m3_decode(it["v_codes_t"][0, 0, :, :N]).T * it["v_scale"][0, 0] + it["v_mean"][0, 0]
    dec = dec_all[200]
    # The other keys keep the exact softmax weight 1 - w200 of the dequantized
    # scores (E4M3 rounding of their P moves it by < 10%); and key 200's code is
    # E4M3(y) = 112 (the running max sits 2 above its score) while the row sum
    # holds y itself, whose exp2 is within the quadratic's 1.963e-3 and whose
    # exponent carries the offset's rounding (half an ulp of B * c + |e|), so
    # the centred output moves by up to that ratio.
    qd = it["q_codes"][0, 0, 5].astype(np.float64) * it["q_scale"][0, 0, 0]
    kd = it["k_codes"][0, 0, :N].astype(np.float64) * np.repeat(it["k_scale"][0, 0], 64)[:N, None]
    s = kd @ qd / 8.0
    w = np.exp(s - s.max())
    w /= w.sum()
    spread = np.abs(dec_all - dec).max(axis=0)
    c = nm.rn32(nm.rn32(np.float64(it["q_scale"][0, 0, 0]) * it["k_scale"][0, 0, 3])
                * np.float64(so.exp2_scale(so.default_sm_scale(D))))
    off = math.log(2) * float(np.spacing(np.float32(float(so.S_BIAS) * float(c) + 64.0))) / 2
    tol = 1.1 * (1 - w[200]) * spread + (1.963e-3 + off) * np.abs(dec - it["v_mean"][0, 0]) + 1e-6
    assert w[200] > 0.999
    assert np.all(np.abs(o[0, 5, 0] - dec) <= tol)


def test_block_scale_indexing_against_exact_attention():
    """Blocks with very different magnitudes: a wrong Q/K block index for a
    scale breaks the agreement with exact attention."""
    rng = np.random.default_rng(18)
    B, N, H, D = 1, 384, 2, 64
    q = rng.standard_normal((B, N, H, D)) * np.repeat(rng.uniform(0.05, 3, (1, N // 64, H, 1)), 64, axis=1)
    k = rng.standard_normal((B, N, H, D)) * np.repeat(rng.uniform(0.05, 3, (1, N // 64, H, 1)), 64, axis=1)
    v = rng.standard_normal((B, N, H, D))
    o, _ = _pipeline(q, k, v)
    qf, kf, vf = (synth.bits_to_f64(_bf16(x)) for x in (q, k, v))
    ex = so.attn_exact_fp64(qf, kf, vf, N)
    cos = (o.ravel() @ ex.ravel()) / np.linalg.norm(o) / np.linalg.norm(ex)
    assert cos >= 0.999


def test_quantized_pipeline_accuracy_gate_tiny():
    """The method's accuracy gate on the tiny workload: cos >= 0.999 vs exact FP64."""
    w = synth.WORKLOADS["tiny"]
    q, k, v = synth.generate(w)
    o, _ = so.sage_pipeline(q, k, v)
    ex = so.attn_exact_fp64(*(synth.bits_to_f64(x) for x in (q, k, v)), w.N)
    cos = (o.ravel() @ ex.ravel()) / np.linalg.norm(o) / np.linalg.norm(ex)
    assert cos >= 0.999


def test_lse_matches_dequantized_logsumexp():
    rng = np.random.default_rng(19)
    B, N, H, D = 1, 200, 1, 64
    q, k, v = (rng.standard_normal((B, N, H, D)) for _ in range(3))
    _, it = _pipeline(q, k, v)
    o, lse = so.attn_fwd(it["q_codes"], it["q_scale"], it["k_codes"], it["k_scale"], it["v_codes_t"],
                         it["v_scale"], it["v_mean"], N, want_lse=True)
    qd = it["q_codes"][0, 0, :N].astype(np.float64) * np.repeat(it["q_scale"][0, 0], 64)[:N, None]
    kd = it["k_codes"][0, 0, :N].astype(np.float64) * np.repeat(it["k_scale"][0, 0], 64)[:N, None]
    s = (qd @ kd.T) / 8.0
    ref = np.log(np.exp(s - s.max(1, keepdims=True)).sum(1)) + s.max(1)
    # l sums weights with relative error <= 1.963e-3 (the quadratic's bound); the
    # rescale factors use the quintic (2.2e-7)
    assert np.abs(lse[0, 0] - ref).max() <= 1.97e-3


def test_two_pass_variant_close_to_online():
    w = synth.WORKLOADS["tiny"]
    q, k, v = synth.generate(w)
    o1, it = so.sage_pipeline(q, k, v)
    o2 = so.attn_fwd(it["q_codes"], it["q_scale"], it["k_codes"], it["k_scale"], it["v_codes_t"],
                     it["v_scale"], it["v_mean"], w.N, two_pass=True)
    cos = (o1.ravel().astype(np.float64) @ o2.ravel()) / np.linalg.norm(o1) / np.linalg.norm(o2)
    assert cos >= 0.999


def test_running_max_with_large_logit_gap():
    """A key in the first tile dominates by ~1000 in exp2 units: the running max
    must carry over tiles (a per-tile max would overflow the rescale)."""
    rng = np.random.default_rng(20)
    B, N, H, D = 1, 384, 1, 64
    q = rng.standard_normal((B, N, H, D)) * 0.01
    k = rng.standard_normal((B, N, H, D)) * 0.01
    q[0, 5, 0] = 10.0
    k[0, 10, 0] = 10.0
    q[0, 5, 0, 1:] = 10.0
    k[0, 10, 0, 1:] = 10.0
    v = rng.standard_normal((B, N, H, D))
    o, it = _pipeline(q, k, v)
    assert np.all(np.isfinite(o))
    dec = nm.e4m3_decode(it["v_codes_t"][0, 0, :, 10]) * it["v_scale"][0, 0] + it["v_mean"][0, 0]
    # The dominant key's exponent is S*c - RN(S*c) + (RN(log2 448 - m) - (log2 448 - m))
    # plus the offset's rounding: off by at most one FP32 ulp of the row max m (here
    # ~1150) and half an ulp of B * c + |e|, and its exp2 is within the quadratic's
    # 1.963e-3, while its code is 112 either way: the centred output moves by up to
    # ln2 * (ulp(m) + ulp(B c + |e|) / 2) + 1.963e-3 relative.
    S = it["q_codes"][0, 0, 5].astype(np.float64) @ it["k_codes"][0, 0, 10].astype(np.float64)
    c = nm.rn32(nm.rn32(np.float64(it["q_scale"][0, 0, 0]) * it["k_scale"][0, 0, 0])
                * np.float64(so.exp2_scale(so.default_sm_scale(D))))
    m = nm.rn32(S * np.float64(c))
    assert m > 512
    centred = np.abs(dec - it["v_mean"][0, 0])                  # the part scaled by P8 / l
    off = float(np.spacing(np.float32(float(so.S_BIAS) * float(c) + 2 * float(m)))) / 2
    tol = (math.log(2) * (np.spacing(np.float32(m)) + off) + 1.963e-3) * centred + 1e-6
    assert np.all(np.abs(o[0, 5, 0] - dec) <= tol)


@pytest.mark.parametrize("coeffs,bound", [(so.EXP2_C, 1.97e-3), (so.EXP2_C5, 2.3e-7)])
def test_exp2_contract_error_bound_and_exact_points(coeffs, bound):
    rng = np.random.default_rng(21)
    u = np.concatenate([rng.uniform(-125, 9.5, 200000), np.arange(-125, 10) + 0.5,
                        np.arange(-125, 10) + 0.4999999, np.linspace(-1, 1, 20001)]).astype(np.float32)
    y = so.exp2_contract(u, coeffs).astype(np.float64)
    rel = np.abs(y / np.exp2(u.astype(np.float64)) - 1)
    assert rel.max() <= bound                                     # the fit's binary32 bound
    n = np.arange(-126, 10).astype(np.float32)
    assert np.array_equal(so.exp2_contract(n, coeffs), np.exp2(n.astype(np.float64)).astype(np.float32))
    lo = so.exp2_contract(np.array([-126.0, -300.0, -np.inf], np.float32), coeffs)
    assert np.all(lo == np.float32(2.0 ** -126))                 # clamped below at 2^-126
    tail = so.exp2_contract(np.linspace(-126, -125, 1001).astype(np.float32), coeffs).astype(np.float64)
    assert np.all((tail >= 0) & (tail < 2.0 ** -124))            # the n = -126 end stays tiny


def test_exp2_contract_coefficients_come_from_the_fit():
    fit_exp2 = pytest.importorskip("oracle.fit_exp2")
    for degree, coeffs in ((2, so.EXP2_C), (5, so.EXP2_C5)):
        assert np.allclose(fit_exp2.fit(degree), np.asarray(coeffs, np.float32), rtol=2e-6, atol=0)
