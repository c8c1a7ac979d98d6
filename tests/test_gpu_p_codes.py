"""The E4M3 codes of P on the GPU, bit for bit against the oracle's.

Every step before the code of y = P~ * 448 is a binary32 operation with a fixed
rounding (the exponent on the biased score, the Cody-Waite split and quadratic
of exp2, the exponent-field add, E4M3 with round-to-nearest-even), so the codes
that the FP8 PV product consumes must equal the oracle's key by key.  The
diagnostic entry point sage_attn_fwd_p_codes runs the same attention and also
writes every code out; its O and LSE must equal sage_attn_fwd's bit for bit.

Cases: a ragged last tile (its masked keys must hold 0), D = 64 and 128,
batch 2, per-token K scales (every tile on per-key multipliers), segment-local
blocks on a joint sequence, all-zero Q (every code is 448), and sampled rows
of two heads at the action-DiT and mid-video sizes.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import sage_oracle as so

pytestmark = pytest.mark.gpu

FILL = 0xA5   # what the P-code buffer holds before the call


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _gpu_p_codes(adt, qb, kb, vb, B, N, H, D, cu=None, q_gran="block64", k_gran="block64"):
    buf = adt.Buffers(B, N, H, D, out_fp32=True, with_lse=True, cu_seqlens=cu, q_gran=q_gran, k_gran=k_gran)
    buf.run(_dev(qb), _dev(kb), _dev(vb))
    pc = torch.full((B * H, N, buf.Npad), FILL, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(buf.out)
    lse = torch.empty_like(buf.lse)
    adt.sage_attn_fwd_p_codes(buf.q_codes, buf.q_scale, buf.k_codes, buf.k_scale, buf.v_codes_t, buf.v_scale,
                              buf.v_mean, buf.shape, 0.0, out, True, pc, lse)
    adt.sage_check()
    assert torch.equal(out.view(torch.int32), buf.out.view(torch.int32))
    assert torch.equal(lse.view(torch.int32), buf.lse.view(torch.int32))
    return buf, pc


def _same_operands(buf, ref_qk, ref_v, b=None, h=None):
    pick = (lambda t: t.cpu().numpy()) if b is None else (lambda t: t[b:b + 1, h:h + 1].cpu().numpy())
    assert np.array_equal(pick(buf.q_codes), ref_qk["q_codes"])
    assert np.array_equal(pick(buf.k_codes), ref_qk["k_codes"])
    assert np.array_equal(pick(buf.q_scale).view(np.uint32), ref_qk["q_scale"].view(np.uint32))
    assert np.array_equal(pick(buf.k_scale).view(np.uint32), ref_qk["k_scale"].view(np.uint32))
    assert np.array_equal(pick(buf.v_codes_t), ref_v["v_codes_t"])


def _oracle_p_codes(ref_qk, ref_v, N, rows=None):
    return so.attn_fwd(ref_qk["q_codes"], ref_qk["q_scale"], ref_qk["k_codes"], ref_qk["k_scale"],
                       ref_v["v_codes_t"], ref_v["v_scale"], ref_v["v_mean"], N, rows=rows,
                       want_p_codes=True)[1]


@pytest.mark.parametrize("B,N,H,D,cu,q_gran,k_gran", [
    (1, 256, 2, 64, None, "block64", "block64"),
    (1, 200, 2, 64, None, "block64", "block64"),
    (2, 1000, 3, 128, None, "block64", "block64"),
    (1, 1000, 2, 128, None, "block64", "token"),
    (1, 1000, 2, 128, (0, 300, 301, 1000), "segment64", "segment64"),
])
def test_p_codes_bit_exact(adt, B, N, H, D, cu, q_gran, k_gran):
    w = synth.custom(B, N, H, D, seed=200 + N, k_sigma=4.0, v_sigma=1.0, outlier_frac=0.02)
    qb, kb, vb = synth.generate(w)
    buf, pc = _gpu_p_codes(adt, qb, kb, vb, B, N, H, D, cu, q_gran, k_gran)
    ref_qk = so.quant_qk(qb, kb, q_gran, k_gran, cu)
    ref_v = so.quant_v(vb)
    _same_operands(buf, ref_qk, ref_v)
    want = _oracle_p_codes(ref_qk, ref_v, N).reshape(B * H, N, N)
    got = pc.cpu().numpy()
    mism = int((got[:, :, :N] != want).sum())
    assert mism == 0, f"{mism} of {want.size} P codes differ"
    assert np.all(got[:, :, N:] == 0)                 # masked keys of the last tile


def test_p_codes_all_zero_q(adt):
    B, N, H, D = 1, 300, 2, 128
    qb, kb, vb = synth.generate(synth.custom(B, N, H, D, seed=211, k_sigma=2.0, v_sigma=1.0))
    qb = np.zeros_like(qb)
    _, pc = _gpu_p_codes(adt, qb, kb, vb, B, N, H, D)
    got = pc.cpu().numpy()
    assert np.all(got[:, :, :N] == 0x7E) and np.all(got[:, :, N:] == 0)


def _rows(N, seed, count=96):
    rng = np.random.default_rng(seed)
    fixed = {0, 1, 127, 128, N - 1, N // 2}
    fixed.update(rng.choice(N, size=count, replace=False).tolist())
    return np.asarray(sorted(fixed), dtype=np.int64)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["action_dit", "mid_video"])
def test_p_codes_full_size_sampled(adt, name):
    w = synth.WORKLOADS[name]
    qb, kb, vb = synth.generate(w)
    buf, pc = _gpu_p_codes(adt, qb, kb, vb, w.B, w.N, w.H, w.D)
    rows = _rows(w.N, w.seed)
    for b, h in [(0, 0), (w.B - 1, w.H - 1)]:
        sl = (slice(b, b + 1), slice(None), slice(h, h + 1), slice(None))
        ref_qk = so.quant_qk(qb[sl], kb[sl])
        ref_v = so.quant_v(vb[sl])
        _same_operands(buf, ref_qk, ref_v, b, h)
        want = _oracle_p_codes(ref_qk, ref_v, w.N, rows)[0, 0]
        got = pc[b * w.H + h][torch.from_numpy(rows).cuda()].cpu().numpy()
        mism = int((got[:, :w.N] != want).sum())
        assert mism == 0, f"{name} head {(b, h)}: {mism} of {want.size} P codes differ"
