"""Parity of sage_quant_qk_normrope (QK RMSNorm + RoPE fused into the INT8
quantization) with the oracle.

Codes, scales and the K mean are bit-exact with the oracle's norm, rotation and
quantization of the same projection outputs; the attention that follows keeps
the gates of the plain path (max-abs 2e-3, cosine >= 0.9999 against the
oracle; cosine >= 0.999 against exact FP64 attention on the normed, rotated
BF16 Q and K).  Cases cover both code kernels and every granularity, ragged
tails, zero and very large token rows, and a full-size workload sampled by head.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import normrope as onr
from oracle import sage_oracle as so

pytestmark = pytest.mark.gpu

ATOL = 2e-3


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _cos(a, b):
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


def _nr_dev(inp):
    return dict(q_w=_dev(inp["q_w"]), k_w=_dev(inp["k_w"]), cos=torch.from_numpy(inp["cos"]).cuda(),
                sin=torch.from_numpy(inp["sin"]).cuda(), eps=inp["eps"])


def _bits32(t):
    return t.cpu().numpy().view(np.uint32)


CASES = [
    # B, N, H, D, q_gran, k_gran, cu_seqlens
    (1, 200, 2, 64, "block64", "block64", None),
    (2, 1000, 3, 128, "block64", "block64", None),
    (1, 384, 2, 128, "token", "block64", None),
    (1, 700, 2, 64, "segment64", "segment64", [0, 37, 37, 190, 520, 700]),
    (1, 130, 1, 128, "token", "token", [0, 3, 5, 130]),
]


@pytest.mark.parametrize("B,N,H,D,q_gran,k_gran,cu", CASES)
def test_normrope_parity(adt, B, N, H, D, q_gran, k_gran, cu):
    w = synth.custom(B, N, H, D, seed=500 + N, k_sigma=4.0, v_sigma=1.0, outlier_frac=0.02,
                     cu_seqlens=tuple(cu) if cu else None)
    q, k = synth.projection_outputs(w)
    _, _, v = synth.generate(w)
    qf = synth.bits_to_f64(q).astype(np.float32)
    qf[0, 1] = 0.0                                        # an all-zero token row
    qf[0, 2] *= 3.0e4                                     # a very large one
    q = synth.to_bf16_bits(qf)
    inp = synth.normrope_inputs(w)
    buf = adt.Buffers(B, N, H, D, out_fp32=True, with_lse=True, cu_seqlens=cu, q_gran=q_gran, k_gran=k_gran)
    buf.run(_dev(q), _dev(k), _dev(v), normrope=_nr_dev(inp))
    adt.sage_check()

    ref = so.quant_qk(q, k, q_gran, k_gran, cu, normrope=inp)
    assert np.array_equal(buf.q_codes.cpu().numpy(), ref["q_codes"])
    assert np.array_equal(_bits32(buf.q_scale), ref["q_scale"].view(np.uint32))
    assert np.array_equal(buf.k_codes.cpu().numpy(), ref["k_codes"])
    assert np.array_equal(_bits32(buf.k_scale), ref["k_scale"].view(np.uint32))
    assert np.array_equal(buf.k_mean.cpu().view(torch.int16).numpy().view(np.uint16), ref["k_mean"])

    rv = so.quant_v(v)
    o32 = buf.out.cpu().numpy()
    o_ref, lse_ref = so.attn_fwd(ref["q_codes"], ref["q_scale"], ref["k_codes"], ref["k_scale"], rv["v_codes_t"],
                                 rv["v_scale"], rv["v_mean"], N, want_lse=True)
    assert np.abs(o32 - o_ref).max() <= ATOL
    assert _cos(o32, o_ref) >= 0.9999
    assert np.abs(buf.lse.cpu().numpy() - lse_ref).max() <= 1e-4 * max(1.0, np.abs(lse_ref).max())
    qn = onr.norm_rope_bf16(q, inp["q_w"], inp["eps"], inp["cos"], inp["sin"])
    kn = onr.norm_rope_bf16(k, inp["k_w"], inp["eps"], inp["cos"], inp["sin"])
    exact = so.attn_exact_fp64(*(synth.bits_to_f64(x) for x in (qn, kn, v)), N)
    assert _cos(o32, exact) >= 0.999


@pytest.mark.slow
def test_normrope_full_size_sampled(adt):
    w = synth.WORKLOADS["action_dit"]
    q, k = synth.projection_outputs(w)
    _, _, v = synth.generate(w)
    inp = synth.normrope_inputs(w)
    buf = adt.Buffers(w.B, w.N, w.H, w.D)
    buf.run(_dev(q), _dev(k), _dev(v), normrope=_nr_dev(inp))
    adt.sage_check()
    for b, h in [(0, 0), (w.B - 1, w.H - 1), (1, 7)]:
        sl = (slice(b, b + 1), slice(None), slice(h, h + 1), slice(None))
        ref = so.quant_qk(q[sl], k[sl], normrope=inp)
        got = lambda t: t[b:b + 1, h:h + 1].cpu().numpy()  # noqa: E731
        assert np.array_equal(got(buf.q_codes), ref["q_codes"])
        assert np.array_equal(got(buf.k_codes), ref["k_codes"])
        assert np.array_equal(got(buf.q_scale).view(np.uint32), ref["q_scale"].view(np.uint32))
        assert np.array_equal(got(buf.k_scale).view(np.uint32), ref["k_scale"].view(np.uint32))
        assert np.array_equal(buf.k_mean[b:b + 1, h:h + 1].cpu().view(torch.int16).numpy().view(np.uint16),
                              ref["k_mean"])
