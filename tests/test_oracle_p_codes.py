"""Pins of the E4M3 codes of P that the oracle records (attn_fwd(want_p_codes=True)).

The codes are the ones the contract feeds to the FP8 PV product ("FLUX.3
Action RTX 5090 report", 02 ENGINEERING, card 03: P quantized to FP8 for the
PV MMA).  They are pinned here against a brute force written from the method's
definition, not from the oracle's loop:

* t = RN32(S * c) with S the exact INT8 dot product and c the score multiplier;
  m_j = the largest t over key tiles 0..j (128 keys each) of the row;
  a key of tile j carries about E4M3(448 * 2^(t - m_j));
* every recorded code is within one E4M3 step of that (the contract's exp2 is
  a quadratic within 2e-3, and its exponent is formed on the biased score),
  and the two agree on nearly all keys;
* the key that sets a tile's running max carries exactly the code of 448;
* recording the codes does not change the output.
"""
import numpy as np
import pytest

import synth
from oracle import numerics as nm
from oracle import sage_oracle as so

TILE = 128


def _operands(B, N, H, D, seed, k_sigma=2.0):
    qb, kb, vb = synth.generate(synth.custom(B, N, H, D, seed=seed, k_sigma=k_sigma, v_sigma=1.0))
    inter = dict(so.quant_qk(qb, kb), **so.quant_v(vb))
    args = (inter["q_codes"], inter["q_scale"], inter["k_codes"], inter["k_scale"], inter["v_codes_t"],
            inter["v_scale"], inter["v_mean"], N)
    return inter, args


def _brute_codes(inter, b, h, N, D):
    """E4M3(448 * 2^(t - m_j)) per (row, key), with m_j the running tile max, in FP64
    from t = RN32(S * c); also returns t and the running max per key."""
    Np = inter["q_codes"].shape[2]
    qc = inter["q_codes"][b, h, :N].astype(np.float64)
    kc = inter["k_codes"][b, h, :N].astype(np.float64)
    S = qc @ kc.T
    qs = np.repeat(inter["q_scale"][b, h], 64)[:N].astype(np.float32)
    ks = np.repeat(inter["k_scale"][b, h], 64)[:N].astype(np.float32)
    sl2e = np.float32(np.float64(np.float32(1.0 / np.sqrt(D))) * np.log2(np.e))
    c = ((qs[:, None] * ks[None, :]).astype(np.float32) * sl2e).astype(np.float32)
    t = (S.astype(np.float32) * c).astype(np.float64)
    m = np.empty_like(t)
    run = np.full(N, -np.inf)
    for j0 in range(0, N, TILE):
        j1 = min(N, j0 + TILE)
        run = np.maximum(run, t[:, j0:j1].max(axis=1))
        m[:, j0:j1] = run[:, None]
    assert Np >= N
    return nm.e4m3_encode((448.0 * np.exp2(t - m)).astype(np.float32)), t, m


@pytest.mark.parametrize("B,N,H,D,seed", [(1, 256, 2, 64, 41), (1, 300, 1, 128, 42), (2, 1000, 1, 64, 43)])
def test_p_codes_follow_the_running_max_definition(B, N, H, D, seed):
    inter, args = _operands(B, N, H, D, seed)
    out, pc = so.attn_fwd(*args, want_p_codes=True)
    assert pc.shape == (B, H, N, N) and pc.dtype == np.uint8
    for b in range(B):
        for h in range(H):
            want, t, m = _brute_codes(inter, b, h, N, D)
            got = pc[b, h]
            assert got.max() <= 0x7E and want.max() <= 0x7E      # positive, finite: codes order like values
            diff = np.abs(got.astype(np.int32) - want.astype(np.int32))
            assert diff.max() <= 1
            assert (diff == 0).mean() >= 0.97
            # the key that sets the running max of its tile carries 448 exactly
            for j0 in range(0, N, TILE):
                j1 = min(N, j0 + TILE)
                tt = t[:, j0:j1]
                setter = tt.max(axis=1) == m[:, j0]
                rows = np.nonzero(setter)[0]
                assert np.all(got[rows, j0 + tt[rows].argmax(axis=1)] == 0x7E)
    # recording is a side output only
    assert np.array_equal(out, so.attn_fwd(*args))


def test_p_codes_of_a_dominant_key_and_of_equal_scores():
    # Q = 0: every score is 0, so every key of every tile carries 448.
    qb, kb, vb = synth.generate(synth.custom(1, 200, 1, 64, seed=44, k_sigma=2.0, v_sigma=1.0))
    inter = dict(so.quant_qk(np.zeros_like(qb), kb), **so.quant_v(vb))
    _, pc = so.attn_fwd(inter["q_codes"], inter["q_scale"], inter["k_codes"], inter["k_scale"],
                        inter["v_codes_t"], inter["v_scale"], inter["v_mean"], 200, want_p_codes=True)
    assert np.all(pc == 0x7E)
    # One key far above the rest in the first tile: it carries 448, the others 0.
    q = np.zeros((1, 130, 1, 64))
    k = np.zeros((1, 130, 1, 64))
    q[0, :, 0, 0] = 8.0
    k[0, :, 0, 0] = -8.0
    k[0, 5, 0, 0] = 8.0
    bits = lambda x: nm.f64_to_bf16_bits(x)
    inter = dict(so.quant_qk(bits(q), bits(k)), **so.quant_v(bits(np.ones((1, 130, 1, 64)))))
    _, pc = so.attn_fwd(inter["q_codes"], inter["q_scale"], inter["k_codes"], inter["k_scale"],
                        inter["v_codes_t"], inter["v_scale"], inter["v_mean"], 130, want_p_codes=True)
    assert np.all(pc[0, 0, :, 5] == 0x7E)
    assert np.all(pc[0, 0, :, :5] == 0) and np.all(pc[0, 0, :, 6:128] == 0)
    # the second tile's keys are measured against the first tile's max, which stays: 0 too
    assert np.all(pc[0, 0, :, 128:] == 0)
