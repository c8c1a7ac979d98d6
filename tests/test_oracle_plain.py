"""Pins of the plain reading of the FP32 online softmax (oracle attn_fwd_plain).

The pages fix INT8 QK, FP8 PV, FP32 accumulation and an FP32 online softmax
("FLUX.3 Action RTX 5090 report", 02 ENGINEERING, card 03; "MiniMax H3 on DGX
Spark", 01 Precision map) and nothing finer.  The plain reading takes those
steps as written: exp2 in FP64 rounded once, no score bias, the running max
exactly the largest score so far, P~ in [0, 1], l from the unquantized P~.
It is pinned here independently of the contract it is used to bound:

* its tile loop with rounding and quantization off equals brute-force FP64
  softmax attention (all tile counts, ragged last tiles, D = 64 and 128);
* closed forms with quantization on: all-zero scores give the mean of the
  dequantized V plus the V mean; one key gives that key's V; a key that
  dominates by a wide margin gives its V;
* the loop written for the contract, run with the plain reading's exp2 and no
  score bias, agrees with this separately written loop;
* on the tiny workload it is as accurate as the method allows against exact
  FP64 attention (cos >= 0.999).
"""
import numpy as np
import pytest

import synth
from oracle import numerics as nm
from oracle import sage_oracle as so


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


@pytest.mark.parametrize("B,N,H,D", [(1, 1, 1, 64), (1, 100, 2, 64), (1, 128, 1, 128), (1, 129, 1, 64),
                                     (2, 300, 2, 64), (1, 1000, 1, 128)])
def test_plain_loop_quant_off_equals_brute_force(B, N, H, D):
    q = _rand((B, N, H, D), 11, 1.5)
    k = _rand((B, N, H, D), 12, 1.5) + _rand((B, 1, H, D), 13, 4)
    v = _rand((B, N, H, D), 14) + _rand((B, 1, H, D), 15, 2)
    ref = so.attn_exact_fp64(q, k, v, N)
    got = so.attn_plain_unquantized(q, k, v, N)
    assert np.abs(got - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


def _quantized_operands(N, D, seed, q_zero=False):
    qb, kb, vb = synth.generate(synth.custom(1, N, 1, D, seed=seed, k_sigma=2.0, v_sigma=1.0))
    if q_zero:
        qb = np.zeros_like(qb)
    inter = dict(so.quant_qk(qb, kb), **so.quant_v(vb))
    return inter, (inter["q_codes"], inter["q_scale"], inter["k_codes"], inter["k_scale"], inter["v_codes_t"],
                   inter["v_scale"], inter["v_mean"], N)


def _dequant_v(inter, N):
    """Dequantized centred V [N, D] (E4M3 decode times the channel scale) in FP64."""
    return (nm.e4m3_decode(inter["v_codes_t"][0, 0, :, :N]).astype(np.float64)
            * inter["v_scale"][0, 0].astype(np.float64)[:, None]).T


@pytest.mark.parametrize("N", [1, 200, 300])
def test_plain_all_equal_scores_give_the_mean_of_v(N):
    # Q = 0: every score is 0, every P~ is exactly 1, every code is 448 and
    # l = N, so the output is the plain mean of the dequantized centred V plus
    # the V mean (to FP32 rounding of the sums).
    inter, args = _quantized_operands(N, 64, seed=21, q_zero=True)
    got = so.attn_fwd_plain(*args)[0, :, 0, :].astype(np.float64)
    want = _dequant_v(inter, N).mean(axis=0) + inter["v_mean"][0, 0]
    assert np.abs(got - want[None, :]).max() <= 2e-6 * max(1.0, np.abs(want).max())


def test_plain_dominant_key_gives_its_v():
    # One key's score exceeds every other by far more than E4M3's range: the
    # others' codes are 0 and their row-sum share is below 2^-40, so every
    # query row returns that key's dequantized V plus the mean.
    N, D = 256, 64
    inter, args = _quantized_operands(N, D, seed=22)
    kc = args[2].copy()
    kc[0, 0, :N] = 0
    kc[0, 0, 77, :] = 127                                # key 77 only
    qc = np.full_like(args[0], 127)
    qc[0, 0, N:] = 0
    q_scale = np.ones_like(args[1])
    k_scale = np.ones_like(args[3])
    got = so.attn_fwd_plain(qc, q_scale, kc, k_scale, *args[4:])[0, :, 0, :].astype(np.float64)
    want = _dequant_v(inter, N)[77] + inter["v_mean"][0, 0]
    assert np.abs(got - want[None, :]).max() <= 1e-6 * max(1.0, np.abs(want).max())


def test_contract_loop_with_plain_exp2_agrees_with_plain_loop():
    # Two separately written loops: the contract's (_attend_rows), given the
    # plain reading's exp2 (FP64, rounded once) and no score bias, and the
    # plain loop.  They still round differently (the contract folds 448 into
    # the exponent and takes its epilogue as one FMA), so an E4M3 code may
    # land on the other side of a rounding boundary; the outputs agree far
    # inside the P quantization error.
    w = synth.WORKLOADS["tiny"]
    qb, kb, vb = synth.generate(w)
    inter = dict(so.quant_qk(qb, kb), **so.quant_v(vb))
    D = w.D
    sl2e = so.exp2_scale(so.default_sm_scale(D))
    for h in range(w.H):
        S = inter["q_codes"][0, h, :w.N].astype(np.float64) @ inter["k_codes"][0, h, :w.N].astype(np.float64).T
        qs = so.token_scales(inter["q_scale"][0, h], so.npad(w.N))[:w.N]
        ks = so.token_scales(inter["k_scale"][0, h], so.npad(w.N))

        def cm(j0, j1):
            return nm.rn32(nm.rn32(qs[:, None].astype(np.float64) * ks[None, j0:j1]) * np.float64(sl2e))

        Vt = nm.e4m3_decode(inter["v_codes_t"][0, h, :, :w.N])
        vs = inter["v_scale"][0, h].astype(np.float64)
        vm = inter["v_mean"][0, h].astype(np.float64)
        o_c, _, _ = so._attend_rows(S, cm, Vt, vs, vm, w.N, nm.rn32, nm.fma32, so._exp2_rn32, so._exp2_rn32,
                                    so._e4m3_round_trip, so.LOG2_P_UNIT)
        o_p, _, _ = so._attend_rows_plain(S, cm, Vt, vs, vm, w.N, nm.rn32, so._exp2_rn32, so._e4m3_round_trip)
        assert np.abs(o_c - o_p).max() <= 1e-4


def test_plain_reading_accuracy_on_tiny():
    w = synth.WORKLOADS["tiny"]
    qb, kb, vb = synth.generate(w)
    o, _ = so.sage_pipeline(qb, kb, vb, plain=True)
    exact = so.attn_exact_fp64(*(synth.bits_to_f64(x) for x in (qb, kb, vb)), w.N)
    a, b = o.astype(np.float64).ravel(), exact.ravel()
    assert a @ b / np.sqrt((a @ a) * (b @ b)) >= 0.999
