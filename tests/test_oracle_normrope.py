"""Pins of the oracle's QK RMSNorm + RoPE step (oracle/normrope.py).

Each check rests on something other than the oracle: values worked out by hand
from the stated order of the FP32 sum, closed forms of the norm and of the
rotation, an FP64 restatement within BF16 rounding, and invariances (per-head
scale, rotation composition) that a wrong axis or a swapped pair would break.
"""
import numpy as np

import synth
from oracle import normrope as nr
from oracle import sage_oracle as so
from oracle.numerics import bf16_bits_to_f32


def _bf(x):
    return synth.to_bf16_bits(np.asarray(x, dtype=np.float32))


def _f(bits):
    return bf16_bits_to_f32(bits)


def test_sum_of_squares_exact_on_small_integers():
    rng = np.random.default_rng(1)
    for D in (64, 128):
        x = rng.integers(-16, 17, size=(5, 3, D)).astype(np.float32)
        assert np.array_equal(nr.sum_of_squares_f32(x), (x.astype(np.int64) ** 2).sum(-1).astype(np.float32))


def test_sum_of_squares_follows_the_stated_order():
    # D = 16: lane 0 holds channels 0-7, lane 1 channels 8-15.  Lane 0 is
    # 2^24 followed by seven 1's: each +1 is a tie that rounds back to 2^24.
    # Lane 1 is eight 1's = 8.  The butterfly gives 2^24 + 8 = 16777224, while
    # the correctly rounded exact sum (2^24 + 15) is 16777232.
    x = np.array([4096.0] + [1.0] * 15, dtype=np.float32)
    assert nr.sum_of_squares_f32(x) == np.float32(16777224.0)
    assert np.float32(2.0 ** 24 + 15) == np.float32(16777232.0)


def test_sum_of_squares_within_the_fp32_bound():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((64, 128)) * rng.uniform(0.01, 100, (64, 1))).astype(np.float32)
    x = _f(_bf(x))
    got = nr.sum_of_squares_f32(x).astype(np.float64)
    exact = (x.astype(np.float64) ** 2).sum(-1)
    assert np.all(np.abs(got - exact) <= 128 * 2.0 ** -24 * exact)


def test_rms_norm_closed_forms():
    D = 64
    ones = _bf(np.ones(D))
    assert np.all(_f(nr.rms_norm_bf16(_bf(np.full((2, D), 2.0)), ones, 0.0)) == 1.0)
    assert np.all(_f(nr.rms_norm_bf16(_bf(np.full((2, D), -8.0)), ones, 0.0)) == -1.0)
    assert np.all(_f(nr.rms_norm_bf16(_bf(np.zeros((2, D))), ones, 1e-6)) == 0.0)
    # weight applied after the normalisation, channel by channel
    w = _bf(np.linspace(0.5, 1.5, D))
    z = _f(nr.rms_norm_bf16(_bf(np.full((1, D), 3.0)), w, 0.0))
    assert np.array_equal(z[0], _f(w))
    # one non-zero channel of value a: mean square a^2 / D, so the output is sqrt(D)
    x = np.zeros((1, D), np.float32)
    x[0, 5] = 0.75
    assert _f(nr.rms_norm_bf16(_bf(x), ones, 0.0))[0, 5] == np.float32(8.0)


def test_rms_norm_against_fp64_formula():
    rng = np.random.default_rng(3)
    D = 128
    x = _bf((rng.standard_normal((4, 50, 3, D)) * np.exp(rng.standard_normal((4, 50, 3, 1)) * 2)))
    w = _bf(1.0 + 0.1 * rng.standard_normal(D))
    eps = float(np.float32(1e-6))
    got = _f(nr.rms_norm_bf16(x, w, eps)).astype(np.float64)
    x64 = _f(x).astype(np.float64)
    ref = x64 / np.sqrt((x64 ** 2).mean(-1, keepdims=True) + eps) * _f(w).astype(np.float64)
    # two BF16 roundings (after the norm, after the weight) plus the FP32 steps
    assert np.all(np.abs(got - ref) <= (2 * 2.0 ** -8 + 1e-6) * np.abs(ref) + 1e-30)


def test_rms_norm_is_per_head_and_scale_free():
    rng = np.random.default_rng(4)
    D = 64
    x = rng.standard_normal((1, 7, 2, D)).astype(np.float32)
    w = _bf(1.0 + 0.1 * rng.standard_normal(D))
    base = nr.rms_norm_bf16(_bf(x), w, 0.0)
    y = x.copy()
    y[:, :, 0] *= 1024.0                                  # head 0 only, by a power of two
    y[:, 3] *= 0.25                                       # one token, both heads
    scaled = nr.rms_norm_bf16(_bf(y), w, 0.0)
    assert np.array_equal(base, scaled)


def test_rope_identity_and_quarter_turn():
    rng = np.random.default_rng(5)
    B, N, H, D = 1, 3, 2, 64
    x = _bf(rng.standard_normal((B, N, H, D)))
    one = np.ones((N, D // 2), np.float32)
    zero = np.zeros((N, D // 2), np.float32)
    assert np.array_equal(nr.rope_bf16(x, one, zero), x)
    q = _f(nr.rope_bf16(x, zero, one))
    xf = _f(x)
    assert np.array_equal(q[..., 0::2], -xf[..., 1::2]) and np.array_equal(q[..., 1::2], xf[..., 0::2])


def test_rope_pairs_adjacent_channels():
    # a unit vector on channel 2i = 6 turned by 0.3 rad at pair i = 3 lands on
    # channels 6 and 7 as (cos 0.3, sin 0.3); the other pairs do not move.
    N, D = 1, 64
    x = np.zeros((1, N, 1, D), np.float32)
    x[..., 6] = 1.0
    cos = np.ones((N, D // 2), np.float32)
    sin = np.zeros((N, D // 2), np.float32)
    cos[0, 3], sin[0, 3] = np.float32(np.cos(0.3)), np.float32(np.sin(0.3))
    cos[0, 4], sin[0, 4] = np.float32(0.0), np.float32(1.0)      # would move channels 8, 9 (zero)
    o = _f(nr.rope_bf16(_bf(x), cos, sin))[0, 0, 0]
    assert o[6] == _f(_bf(np.cos(0.3))) and o[7] == _f(_bf(np.sin(0.3)))
    assert not np.delete(o, [6, 7]).any()


def test_rope_keeps_pair_norms_and_composes():
    rng = np.random.default_rng(6)
    N, D = 40, 128
    x = _bf(rng.standard_normal((1, N, 2, D)))
    a1 = rng.uniform(-3, 3, (N, D // 2))
    a2 = rng.uniform(-3, 3, (N, D // 2))
    t = lambda a: (np.cos(a).astype(np.float32), np.sin(a).astype(np.float32))  # noqa: E731
    once = _f(nr.rope_bf16(x, *t(a1 + a2))).astype(np.float64)
    twice = _f(nr.rope_bf16(nr.rope_bf16(x, *t(a1)), *t(a2))).astype(np.float64)
    xf = _f(x).astype(np.float64)
    n_in = xf[..., 0::2] ** 2 + xf[..., 1::2] ** 2
    n_out = once[..., 0::2] ** 2 + once[..., 1::2] ** 2
    assert np.all(np.abs(np.sqrt(n_out) - np.sqrt(n_in)) <= 2 * 2.0 ** -8 * np.sqrt(n_in) + 1e-30)
    mag = np.repeat(np.sqrt(n_in), 2, axis=-1)
    assert np.all(np.abs(once - twice) <= 4 * 2.0 ** -8 * mag + 1e-30)


def test_rope_tables_layout():
    D = 128
    pairs = synth.rope_axes(D)
    assert sum(pairs) == D // 2
    pos = np.zeros((3, 4), np.int64)
    pos[1, 0] = 1                                        # t = 1
    pos[2, 3] = 5                                        # l = 5
    cos, sin = synth.rope_tables(pos, D)
    assert np.all(cos[0] == 1) and np.all(sin[0] == 0)
    # t = 1: the first 16 pairs turn by 10000^(-j/16) rad, the rest stay
    j = np.arange(pairs[0])
    assert np.array_equal(cos[1, :16], np.cos(10000.0 ** (-j / 16)).astype(np.float32))
    assert np.all(cos[1, 16:] == 1) and np.all(sin[1, 16:] == 0)
    # l = 5: only the last 16 pairs move, pair 48 by 5 rad
    assert np.all(sin[2, :48] == 0) and sin[2, 48] == np.float32(np.sin(5.0))


def test_quant_qk_with_normrope_is_quant_of_the_normed_rotated_bf16():
    w = synth.custom(1, 200, 2, 64, seed=11, k_sigma=3.0, v_sigma=1.0)
    q, k = synth.projection_outputs(w)
    inp = synth.normrope_inputs(w)
    fused = so.quant_qk(q, k, normrope=inp)
    qn = nr.norm_rope_bf16(q, inp["q_w"], inp["eps"], inp["cos"], inp["sin"])
    kn = nr.norm_rope_bf16(k, inp["k_w"], inp["eps"], inp["cos"], inp["sin"])
    plain = so.quant_qk(qn, kn)
    for key in ("q_codes", "q_scale", "k_codes", "k_scale", "k_mean"):
        assert np.array_equal(fused[key], plain[key]), key
    # the norm removes per-token scale: power-of-two rescaled tokens give the same codes
    qf = synth.bits_to_f64(q).astype(np.float32)
    qf[:, ::3] *= 64.0
    again = so.quant_qk(synth.to_bf16_bits(qf), k, normrope=dict(inp, eps=0.0))
    ref = so.quant_qk(q, k, normrope=dict(inp, eps=0.0))
    assert np.array_equal(again["q_codes"], ref["q_codes"])


def test_parity_case_can_tell_a_fused_rotation_apart():
    """The D = 128 GPU parity case holds rotations that land within an ulp of a
    BF16 midpoint, where RN(RN(c*a) - RN(s*b)) and a fused multiply-add
    (RN(c*a - RN(s*b)), one rounding fewer) round to different BF16 values, so
    that case would catch a kernel whose rotation got fused."""
    w = synth.custom(2, 1000, 3, 128, seed=1500, k_sigma=4.0, v_sigma=1.0, outlier_frac=0.02)
    q, _ = synth.projection_outputs(w)
    inp = synth.normrope_inputs(w)
    z = _f(nr.rms_norm_bf16(q, inp["q_w"], inp["eps"])).astype(np.float64)
    c = inp["cos"][None, :, None, :].astype(np.float64)
    s = inp["sin"][None, :, None, :].astype(np.float64)
    a, b = z[..., 0::2], z[..., 1::2]
    sep = (np.float32(c * a) - np.float32(s * b)).astype(np.float32)
    fused = (c * a - np.float32(s * b).astype(np.float64)).astype(np.float32)
    assert np.count_nonzero(_bf(sep) != _bf(fused)) >= 1
