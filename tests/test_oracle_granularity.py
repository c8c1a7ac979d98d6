"""Pins of the oracle's INT8 scale granularities (64-token blocks, one scale per
token, 64-token blocks local to each segment of a packed joint sequence).

Each check rests on something other than the oracle itself: group boundaries
written out by hand from the definition, a pure-Python loop over every group
with exact rational rounding, orderings that must hold between granularities,
and cases where two granularities must coincide.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import synth
from oracle import sage_oracle as so


def test_scale_groups_written_out():
    assert so.scale_groups(200, "block64").tolist() == [0, 64, 128, 192]
    assert so.scale_groups(200, "token").tolist() == list(range(256))
    # segments [0, 10), [10, 150), [150, 200); padding [200, 256)
    assert so.scale_groups(200, "segment64", [0, 10, 150, 200]).tolist() == [0, 10, 74, 138, 150, 200]
    # no cu_seqlens: one segment, so the blocks are the global grid up to N
    assert so.scale_groups(130, "segment64").tolist() == [0, 64, 128, 130, 194]
    # empty segments add nothing
    assert so.scale_groups(128, "segment64", [0, 0, 64, 64, 128]).tolist() == [0, 64]
    with pytest.raises(ValueError):
        so.scale_groups(10, "per-warp")


@pytest.mark.parametrize("seed", range(5))
def test_segment_blocks_cover_the_axis_and_never_cross_a_segment(seed):
    rng = np.random.default_rng(seed)
    N = int(rng.integers(1, 3000))
    cuts = np.sort(rng.integers(0, N + 1, size=int(rng.integers(0, 6))))
    cu = [0] + cuts.tolist() + [N]
    starts = so.scale_groups(N, "segment64", cu)
    Np = so.npad(N)
    ends = np.append(starts[1:], Np)
    assert starts[0] == 0 and np.all(ends > starts) and np.all(ends - starts <= 64)
    for a in cu[:-1]:
        if a < N:
            assert a in starts                           # every non-empty segment starts a block
    bounds = np.asarray(cu + [Np])
    for s, e in zip(starts, ends):
        seg = np.searchsorted(bounds, s, side="right") - 1
        assert e <= max(bounds[seg + 1], N if s < N else Np)   # inside one segment (or the padding)
        if s < N:
            assert e <= N


def _brute_group(xg):
    """The INT8 rule on one group, from the definition, in exact rationals."""
    amax = max(abs(Fraction(float(v))) for v in xg.ravel())
    if amax == 0:
        return 0.0, np.zeros(xg.shape, dtype=np.int8), None
    scale = float(np.float32(float(amax) / 127.0))
    ideal = np.vectorize(lambda v: float(Fraction(float(v)) * 127 / amax))(xg.astype(np.float64))
    return scale, None, ideal


@pytest.mark.parametrize("gran,cu", [("token", None), ("segment64", [0, 37, 37, 190, 200]),
                                     ("segment64", None)])
def test_group_quant_brute_force(gran, cu):
    rng = np.random.default_rng(hash(gran) % 1000)
    N, D = 200, 16
    x = (rng.standard_normal((1, 2, so.npad(N), D)) * rng.uniform(0.01, 40, (1, 2, so.npad(N), 1)))
    x = x.astype(np.float32)
    x[:, :, N:] = 0.0
    x[0, 1, 40:45] = 0.0                                 # zero tokens (a zero group in token mode)
    codes, scale = so.quant_scales(x, N, gran, cu)
    assert scale.shape == (1, 2, so.npad(N)) and codes.shape == x.shape
    starts = so.scale_groups(N, gran, cu)
    ends = np.append(starts[1:], x.shape[2])
    for h in range(2):
        for s, e in zip(starts, ends):
            bscale, zero_codes, ideal = _brute_group(x[0, h, s:e])
            assert np.all(scale[0, h, s:e] == np.float32(bscale))
            cg = codes[0, h, s:e]
            if zero_codes is not None:
                assert not cg.any()
                continue
            assert np.abs(cg).max() == 127
            frac = np.abs(ideal - np.floor(ideal) - 0.5)
            ok = frac > 1e-4                             # away from a rounding tie
            assert np.array_equal(cg[ok], np.rint(ideal[ok]).astype(np.int8))
            assert np.all(np.abs(cg[~ok] - ideal[~ok]) <= 0.5 + 1e-4)


def test_token_scale_never_coarser_than_its_block():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((2, 3, 256, 32)) * rng.uniform(0.1, 9, (2, 3, 256, 1))).astype(np.float32)
    _, sb = so.quant_scales(x, 256, "block64")
    ct, st = so.quant_scales(x, 256, "token")
    sbt = np.repeat(sb, 64, axis=2)
    assert np.all(st <= sbt)
    # the token holding its block's absmax has the block's scale
    amax_tok = np.abs(x).max(axis=3)
    holder = amax_tok == np.repeat(amax_tok.reshape(2, 3, 4, 64).max(axis=3), 64, axis=2)
    assert np.array_equal(st[holder], sbt[holder])
    # per-token reconstruction error within half a step of the token's own scale
    err = np.abs(ct.astype(np.float64) * st[..., None] - x)
    assert np.all(err <= st[..., None].astype(np.float64) * (0.5 + 2.0 ** -20))


def test_equal_token_absmax_makes_token_and_block_identical():
    rng = np.random.default_rng(4)
    base = rng.standard_normal(32).astype(np.float32)
    # every token: a signed permutation of one vector, so all absmaxes are equal
    x = np.stack([rng.permutation(base) * rng.choice([-1, 1], 32) for _ in range(128)]).astype(np.float32)
    x = x[None, None]
    cb, sb = so.quant_scales(x, 128, "block64")
    ct, st = so.quant_scales(x, 128, "token")
    assert np.array_equal(cb, ct) and np.array_equal(np.repeat(sb, 64, axis=2), st)


def test_aligned_segments_give_the_block_grid():
    rng = np.random.default_rng(5)
    N = 640
    x = rng.standard_normal((1, 2, N, 16)).astype(np.float32)
    cb, sb = so.quant_scales(x, N, "block64")
    cs, ss = so.quant_scales(x, N, "segment64", [0, 128, 512, 640])
    assert np.array_equal(cb, cs) and np.array_equal(np.repeat(sb, 64, axis=2), ss)
    # a misaligned cut changes the blocks around it, and only those
    cm, sm = so.quant_scales(x, N, "segment64", [0, 100, 640])
    same = np.repeat(sb, 64, axis=2) == sm
    assert same[:, :, :64].all() and not same[:, :, 64:128].all()


def test_attention_reads_both_scale_layouts_alike():
    q, k, v = synth.generate(synth.custom(1, 300, 2, 64, seed=8, k_sigma=3.0, v_sigma=1.0))
    qk = so.quant_qk(q, k)
    vv = so.quant_v(v)
    Np = so.npad(300)
    args = (qk["k_codes"],)
    o_blk = so.attn_fwd(qk["q_codes"], qk["q_scale"], qk["k_codes"], qk["k_scale"], vv["v_codes_t"],
                        vv["v_scale"], vv["v_mean"], 300)
    o_tok = so.attn_fwd(qk["q_codes"], np.repeat(qk["q_scale"], 64, axis=2), *args,
                        np.repeat(qk["k_scale"], 64, axis=2), vv["v_codes_t"], vv["v_scale"],
                        vv["v_mean"], 300)
    assert np.array_equal(o_blk, o_tok)
    assert so.token_scales(qk["q_scale"][0, 0], Np).shape == (Np,)


def _cos(a, b):
    a = a.astype(np.float64).ravel()
    b = b.astype(np.float64).ravel()
    return float(a @ b / math.sqrt((a @ a) * (b @ b)))


@pytest.mark.parametrize("N,D", [(256, 64), (512, 128)])
def test_token_q_scales_help_when_some_rows_are_large(N, D):
    # 1 query row in 32 is 20x larger: with 64-token blocks it sets the scale of
    # its whole block, so the other rows keep only a few INT8 levels.
    B, H = 1, 2
    q, k, v = synth.generate(synth.custom(B, N, H, D, seed=9, k_sigma=2.0, v_sigma=1.0))
    qf = synth.bits_to_f64(q).astype(np.float32)
    qf[:, ::32] *= 20.0
    q = synth.to_bf16_bits(qf)
    exact = so.attn_exact_fp64(synth.bits_to_f64(q), synth.bits_to_f64(k), synth.bits_to_f64(v), N)
    o_blk, _ = so.sage_pipeline(q, k, v)
    o_tok, _ = so.sage_pipeline(q, k, v, q_gran="token")
    small = np.ones(N, dtype=bool)
    small[::32] = False                                  # the rows that share a block with a large one
    err_blk = np.abs(o_blk - exact)[:, small].max()
    err_tok = np.abs(o_tok - exact)[:, small].max()
    assert err_tok < 0.5 * err_blk
    assert _cos(o_tok[:, small], exact[:, small]) > _cos(o_blk[:, small], exact[:, small])
