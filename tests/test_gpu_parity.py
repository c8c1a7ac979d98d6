"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Quantization outputs (codes, scales, means) must be bit-exact.  The attention
output (FP32) must be within max-abs 2e-3 and cosine >= 0.9999 of the oracle,
and cosine >= 0.999 of exact FP64 attention on the BF16 inputs; the BF16
output must be the RNE rounding of the FP32 output.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import numerics as nm
from oracle import sage_oracle as so

pytestmark = pytest.mark.gpu

ATOL = 2e-3
COS_ORACLE = 0.9999
COS_EXACT = 0.999


def _dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _cos(a, b):
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


def _run_quant(adt, q, k, v, B, N, H, D, tok_stride=0, v_tok_stride=0):
    buf = adt.Buffers(B, N, H, D, out_fp32=True, with_lse=True, tok_stride=tok_stride)
    vshape = adt.make_shape(B, N, H, D, v_tok_stride) if v_tok_stride else None
    adt.sage_quant_qk(q, k, buf.shape, buf.q_codes, buf.q_scale, buf.k_codes, buf.k_scale, buf.k_mean,
                      buf.workspace)
    adt.sage_quant_v(v, vshape or buf.shape, buf.v_codes_t, buf.v_scale, buf.v_mean, buf.workspace)
    adt.sage_check()
    return buf


def _bits32(t):
    return t.cpu().numpy().view(np.uint32)


def _check_quant(buf, ref_qk, ref_v):
    assert np.array_equal(buf.q_codes.cpu().numpy(), ref_qk["q_codes"])
    assert np.array_equal(_bits32(buf.q_scale), ref_qk["q_scale"].view(np.uint32))
    assert np.array_equal(buf.k_mean.cpu().view(torch.int16).numpy().view(np.uint16), ref_qk["k_mean"])
    assert np.array_equal(buf.k_codes.cpu().numpy(), ref_qk["k_codes"])
    assert np.array_equal(_bits32(buf.k_scale), ref_qk["k_scale"].view(np.uint32))
    assert np.array_equal(_bits32(buf.v_mean), ref_v["v_mean"].view(np.uint32))
    assert np.array_equal(_bits32(buf.v_scale), ref_v["v_scale"].view(np.uint32))
    assert np.array_equal(buf.v_codes_t.cpu().numpy(), ref_v["v_codes_t"])


SHAPES = [
    (1, 256, 2, 64),     # tiny workload shape
    (1, 1, 2, 64),       # a single token
    (1, 65, 3, 128),     # one full block plus one token
    (1, 200, 2, 64),     # ragged last tile
    (2, 1000, 3, 128),   # several tiles, ragged, batch 2
    (1, 1536, 4, 128),   # 12 KV tiles, odd head count of blocks
]


@pytest.mark.parametrize("B,N,H,D", SHAPES)
def test_quant_and_attention_parity(adt, B, N, H, D):
    w = synth.custom(B, N, H, D, seed=100 + N, k_sigma=4.0, v_sigma=1.0, outlier_frac=0.02)
    qb, kb, vb = synth.generate(w)
    buf = _run_quant(adt, _dev(qb), _dev(kb), _dev(vb), B, N, H, D)
    ref_qk = so.quant_qk(qb, kb)
    ref_v = so.quant_v(vb)
    _check_quant(buf, ref_qk, ref_v)

    adt.sage_attn_fwd(buf.q_codes, buf.q_scale, buf.k_codes, buf.k_scale, buf.v_codes_t, buf.v_scale,
                      buf.v_mean, buf.shape, 0.0, buf.out, True, buf.lse)
    adt.sage_check()
    o32 = buf.out.cpu().numpy()
    ref, lse_ref = so.attn_fwd(ref_qk["q_codes"], ref_qk["q_scale"], ref_qk["k_codes"], ref_qk["k_scale"],
                               ref_v["v_codes_t"], ref_v["v_scale"], ref_v["v_mean"], N, want_lse=True)
    assert np.all(np.isfinite(o32))
    assert np.abs(o32 - ref).max() <= ATOL
    assert _cos(o32, ref) >= COS_ORACLE
    assert np.abs(buf.lse.cpu().numpy() - lse_ref).max() <= 1e-4 * max(1.0, np.abs(lse_ref).max())
    exact = so.attn_exact_fp64(*(synth.bits_to_f64(x) for x in (qb, kb, vb)), N)
    assert _cos(o32, exact) >= COS_EXACT

    # BF16 output = RNE(FP32 output), from a separate call
    o16 = torch.empty((B, N, H, D), dtype=torch.bfloat16, device="cuda")
    adt.sage_attn_fwd(buf.q_codes, buf.q_scale, buf.k_codes, buf.k_scale, buf.v_codes_t, buf.v_scale,
                      buf.v_mean, buf.shape, 0.0, o16, False, None)
    adt.sage_check()
    assert np.array_equal(o16.cpu().view(torch.int16).numpy().view(np.uint16), nm.f32_to_bf16_bits(o32))


def test_tiny_workload_and_determinism(adt):
    w = synth.WORKLOADS["tiny"]
    qb, kb, vb = synth.generate(w)
    q, k, v = _dev(qb), _dev(kb), _dev(vb)
    buf = adt.Buffers(w.B, w.N, w.H, w.D, out_fp32=True)
    o1 = buf.run(q, k, v).clone()
    codes1 = (buf.q_codes.clone(), buf.k_codes.clone(), buf.v_codes_t.clone())
    o2 = buf.run(q, k, v).clone()
    adt.sage_check()
    assert torch.equal(o1, o2)
    assert all(torch.equal(a, b) for a, b in zip(codes1, (buf.q_codes, buf.k_codes, buf.v_codes_t)))
    ref, _ = so.sage_pipeline(qb, kb, vb)
    assert np.abs(o1.cpu().numpy() - ref).max() <= ATOL


def test_strided_v_and_q_k_inputs(adt):
    """V read in place from a wider projection output (token stride > H*D)."""
    B, N, H, D = 1, 300, 2, 128
    w = synth.custom(B, N, H, D, seed=7, v_sigma=1.0)
    qb, kb, vb = synth.generate(w)
    wide = np.zeros((B, N, H * D + 512), np.uint16)
    wide[:, :, 256:256 + H * D] = vb.reshape(B, N, H * D)
    wide_dev = _dev(wide)
    v_view = wide_dev[:, :, 256:256 + H * D]
    buf = _run_quant(adt, _dev(qb), _dev(kb), v_view, B, N, H, D, v_tok_stride=H * D + 512)
    _check_quant(buf, so.quant_qk(qb, kb), so.quant_v(vb))
    # strided Q and K as well
    wq = np.zeros((B, N, H * D + 64), np.uint16)
    wq[:, :, :H * D] = qb.reshape(B, N, H * D)
    wk = np.zeros((B, N, H * D + 64), np.uint16)
    wk[:, :, :H * D] = kb.reshape(B, N, H * D)
    buf2 = _run_quant(adt, _dev(wq), _dev(wk), _dev(vb), B, N, H, D, tok_stride=H * D + 64, v_tok_stride=H * D)
    _check_quant(buf2, so.quant_qk(qb, kb), so.quant_v(vb))


def test_degenerate_inputs(adt):
    """All-zero Q (uniform softmax), constant V (zero centred V, zero scales)."""
    B, N, H, D = 1, 192, 2, 64
    rng = np.random.default_rng(3)
    qb = synth.to_bf16_bits(np.zeros((B, N, H, D), np.float32))
    kb = synth.to_bf16_bits(rng.standard_normal((B, N, H, D)).astype(np.float32))
    vb = synth.to_bf16_bits(np.full((B, N, H, D), 1.5, np.float32))
    buf = _run_quant(adt, _dev(qb), _dev(kb), _dev(vb), B, N, H, D)
    _check_quant(buf, so.quant_qk(qb, kb), so.quant_v(vb))
    assert float(buf.v_scale.abs().max()) == 0.0
    adt.sage_attn_fwd(buf.q_codes, buf.q_scale, buf.k_codes, buf.k_scale, buf.v_codes_t, buf.v_scale,
                      buf.v_mean, buf.shape, 0.0, buf.out, True, None)
    adt.sage_check()
    assert torch.all(buf.out == 1.5)


def test_explicit_sm_scale(adt):
    B, N, H, D = 1, 384, 2, 128
    w = synth.custom(B, N, H, D, seed=9)
    qb, kb, vb = synth.generate(w)
    buf = _run_quant(adt, _dev(qb), _dev(kb), _dev(vb), B, N, H, D)
    adt.sage_attn_fwd(buf.q_codes, buf.q_scale, buf.k_codes, buf.k_scale, buf.v_codes_t, buf.v_scale,
                      buf.v_mean, buf.shape, 0.05, buf.out, True, None)
    adt.sage_check()
    ref, inter = so.sage_pipeline(qb, kb, vb, sm_scale=0.05)
    assert np.abs(buf.out.cpu().numpy() - ref).max() <= ATOL


def test_wait_timeout_is_reported_and_context_survives(adt):
    adt.selftest_wait_timeout(2_000_000)      # 2 ms on a barrier nothing completes
    assert adt.sage_check_status() == 5        # SAGE_ERR_DEVICE_TIMEOUT
    assert adt.sage_check_status() == 0        # cleared
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0


@pytest.mark.parametrize("B,N,H,D", [(1, 200, 2, 64), (2, 1000, 3, 128), (1, 4096, 24, 128)])
def test_fused_qkv_quantization_equals_the_two_calls(adt, B, N, H, D):
    """sage_quant_qkv writes the same bytes as sage_quant_qk + sage_quant_v,
    with a strided V as well."""
    w = synth.custom(B, N, H, D, seed=40 + N, k_sigma=4.0, v_sigma=1.0, outlier_frac=0.02)
    qb, kb, vb = synth.generate(w)
    wide = np.zeros((B, N, H * D + 64), np.uint16)
    wide[:, :, 32:32 + H * D] = vb.reshape(B, N, H * D)
    v_view = _dev(wide)[:, :, 32:32 + H * D]
    sep = _run_quant(adt, _dev(qb), _dev(kb), v_view, B, N, H, D, v_tok_stride=H * D + 64)
    fused = adt.Buffers(B, N, H, D, out_fp32=True)
    adt.sage_quant_qkv(_dev(qb), _dev(kb), v_view, fused.shape, H * D + 64, fused.q_codes, fused.q_scale,
                       fused.k_codes, fused.k_scale, fused.k_mean, fused.v_codes_t, fused.v_scale, fused.v_mean,
                       fused.workspace)
    adt.sage_check()
    for name in ("q_codes", "q_scale", "k_codes", "k_scale", "k_mean", "v_codes_t", "v_scale", "v_mean"):
        assert torch.equal(getattr(sep, name), getattr(fused, name)), name
    _check_quant(fused, so.quant_qk(qb, kb), so.quant_v(vb))
