"""Parity of the CUDA path with the oracle at the finer INT8 scale granularities:
one Q or K scale per token, and 64-token blocks local to each segment of a
packed joint sequence.

Codes and scales bit-exact; attention within the same bounds as the 64-token
block path (max-abs 2e-3 and cosine >= 0.9999 against the oracle, cosine >=
0.999 against exact FP64 attention).  The cases cover both kernels of the Q/K
code pass (a tensor at block granularity next to one at a finer one), tiles
whose K scales are equal within each 64-key half and tiles that mix them,
empty and very short segments, and ragged last tiles.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import sage_oracle as so

pytestmark = pytest.mark.gpu

ATOL = 2e-3
COS_ORACLE = 0.9999
COS_EXACT = 0.999

CASES = [
    # B, N, H, D, q_gran, k_gran, cu_seqlens
    (1, 200, 2, 64, "token", "block64", None),
    (2, 1000, 3, 128, "token", "block64", None),
    (1, 1000, 2, 128, "block64", "token", None),
    (1, 700, 2, 64, "segment64", "segment64", [0, 37, 37, 190, 520, 700]),
    (1, 1536, 2, 128, "token", "segment64", [0, 512, 1500, 1536]),
    (1, 130, 1, 64, "segment64", "token", [0, 3, 5, 130]),
    (2, 384, 2, 128, "token", "token", None),
]


def _dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _cos(a, b):
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


def _bits32(t):
    return t.cpu().numpy().view(np.uint32)


@pytest.mark.parametrize("B,N,H,D,q_gran,k_gran,cu", CASES)
def test_granularity_parity(adt, B, N, H, D, q_gran, k_gran, cu):
    w = synth.custom(B, N, H, D, seed=300 + N, k_sigma=4.0, v_sigma=1.0, outlier_frac=0.02)
    qb, kb, vb = synth.generate(w)
    buf = adt.Buffers(B, N, H, D, out_fp32=True, with_lse=True, cu_seqlens=cu, q_gran=q_gran, k_gran=k_gran)
    # poison the outputs: every byte must be written by the call
    for t in (buf.q_codes, buf.k_codes):
        t.fill_(0x55)
    for t in (buf.q_scale, buf.k_scale):
        t.fill_(float("nan"))
    buf.run(_dev(qb), _dev(kb), _dev(vb))
    adt.sage_check()

    ref_qk = so.quant_qk(qb, kb, q_gran, k_gran, cu)
    assert np.array_equal(buf.q_codes.cpu().numpy(), ref_qk["q_codes"])
    assert np.array_equal(_bits32(buf.q_scale), ref_qk["q_scale"].view(np.uint32))
    assert np.array_equal(buf.k_codes.cpu().numpy(), ref_qk["k_codes"])
    assert np.array_equal(_bits32(buf.k_scale), ref_qk["k_scale"].view(np.uint32))

    ref_v = so.quant_v(vb)
    o32 = buf.out.cpu().numpy()
    ref, lse_ref = so.attn_fwd(ref_qk["q_codes"], ref_qk["q_scale"], ref_qk["k_codes"], ref_qk["k_scale"],
                               ref_v["v_codes_t"], ref_v["v_scale"], ref_v["v_mean"], N, want_lse=True)
    assert np.all(np.isfinite(o32))
    assert np.abs(o32 - ref).max() <= ATOL
    assert _cos(o32, ref) >= COS_ORACLE
    assert np.abs(buf.lse.cpu().numpy() - lse_ref).max() <= 1e-4 * max(1.0, np.abs(lse_ref).max())
    exact = so.attn_exact_fp64(*(synth.bits_to_f64(x) for x in (qb, kb, vb)), N)
    assert _cos(o32, exact) >= COS_EXACT


def test_per_token_q_beats_blocks_on_large_rows(adt):
    """On the GPU path too: rows that share a block with a 20x larger row come
    out closer to exact attention with one Q scale per token."""
    B, N, H, D = 1, 512, 2, 128
    qb, kb, vb = synth.generate(synth.custom(B, N, H, D, seed=9, k_sigma=2.0, v_sigma=1.0))
    qf = synth.bits_to_f64(qb).astype(np.float32)
    qf[:, ::32] *= 20.0
    qb = synth.to_bf16_bits(qf)
    exact = so.attn_exact_fp64(*(synth.bits_to_f64(x) for x in (qb, kb, vb)), N)
    small = np.ones(N, dtype=bool)
    small[::32] = False
    errs = {}
    for gran in ("block64", "token"):
        buf = adt.Buffers(B, N, H, D, out_fp32=True, q_gran=gran)
        buf.run(_dev(qb), _dev(kb), _dev(vb))
        adt.sage_check()
        errs[gran] = np.abs(buf.out.cpu().numpy() - exact)[:, small].max()
    assert errs["token"] < 0.5 * errs["block64"]
