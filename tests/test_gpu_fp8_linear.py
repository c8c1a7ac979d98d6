"""Parity of the row-wise FP8 projection (sage_fp8_quant_rows, sage_fp8_linear)
with the oracle.

The quantizer is bit-exact.  The product accumulates in FP32 on the tensor
cores in their own order, so the FP32 output is held to the bound that any
FP32 summation order meets: |y - y_ref| <= (K * 2^-24 * sum_k |x_k w_k|) * sx
* sw (the accumulation) + 2 ulp(y) (the two rounded scale products on each
side).  The BF16 output equals RN_bf16 of the FP32 output bit for bit.
Shapes cover one tile, ragged M / N / K tails, several waves of the persistent
grid, a last wave split into 4 and into 2 column blocks per tile, and full-size
projections of the action-DiT workload (sampled rows; the MLP down-projection
splits its last wave).
"""
import numpy as np
import pytest
import torch

import synth
from oracle import fp8_linear as fl
from oracle.numerics import e4m3_decode, f32_to_bf16_bits

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _inputs(M, N, K, seed):
    rng = np.random.default_rng(seed)
    x = synth.to_bf16_bits((rng.standard_normal((M, K)) * np.exp(rng.standard_normal((M, 1)))).astype(np.float32))
    w = synth.to_bf16_bits((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    return x, w


def _quant(adt, bits):
    R, K = bits.shape
    codes = torch.empty((R, K), dtype=torch.uint8, device="cuda")
    scale = torch.empty(R, dtype=torch.float32, device="cuda")
    adt.sage_fp8_quant_rows(_dev(bits), codes, scale)
    return codes, scale


def _bound(xq, sx, wq, sw, y_ref, rows=None):
    rows = np.arange(xq.shape[0]) if rows is None else rows
    ax = np.abs(e4m3_decode(xq[rows]))
    aw = np.abs(e4m3_decode(wq))
    K = xq.shape[1]
    acc_err = K * 2.0 ** -24 * (ax @ aw.T)
    return acc_err * sx[rows, None].astype(np.float64) * sw[None, :].astype(np.float64) + \
        2 * np.spacing(np.abs(y_ref).astype(np.float32)).astype(np.float64)


@pytest.mark.parametrize("R,K,ld", [(1, 8, 8), (7, 264, 264), (33, 3072, 3200), (5, 16384, 16384)])
def test_quant_rows_bit_exact(adt, R, K, ld):
    rng = np.random.default_rng(R * K)
    full = synth.to_bf16_bits((rng.standard_normal((R, ld)) * np.exp(3 * rng.standard_normal((R, 1)))).astype(np.float32))
    full[0, :K] = 0                                        # a zero row
    xd = _dev(full)[:, :K]
    codes = torch.empty((R, K), dtype=torch.uint8, device="cuda")
    scale = torch.empty(R, dtype=torch.float32, device="cuda")
    adt.sage_fp8_quant_rows(xd, codes, scale)
    adt.sage_check()
    rc, rs = fl.fp8_quant_rows(full[:, :K])
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(scale.cpu().numpy().view(np.uint32), rs.view(np.uint32))


# (4736, 1280, 4224): 185 tiles of 128 x 256 on 148 SMs, the last 37 as 4 column blocks each;
# (6656, 1024, 4224): 208 tiles, the last 60 as 2 column blocks each.
@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (300, 264, 272), (1000, 1536, 1024), (130, 8, 4096),
                                   (4736, 1280, 4224), (6656, 1024, 4224)])
def test_fp8_linear_parity(adt, M, N, K):
    x, w = _inputs(M, N, K, seed=M + N + K)
    xq, sx = _quant(adt, x)
    wq, sw = _quant(adt, w)
    out32 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    adt.sage_fp8_linear(xq, sx, wq, sw, out32)
    out16 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    adt.sage_fp8_linear(xq, sx, wq, sw, out16)
    adt.sage_check()
    xq_h, sx_h, wq_h, sw_h = (t.cpu().numpy() for t in (xq, sx, wq, sw))
    ref = fl.fp8_linear(xq_h, sx_h, wq_h, sw_h)
    y = out32.cpu().numpy()
    assert np.all(np.isfinite(y))
    assert np.all(np.abs(y.astype(np.float64) - ref) <= _bound(xq_h, sx_h, wq_h, sw_h, ref))
    assert np.array_equal(out16.cpu().view(torch.int16).numpy().view(np.uint16), f32_to_bf16_bits(y))


@pytest.mark.slow
@pytest.mark.parametrize("M,N,K", [(8192, 12288, 3072), (8192, 3072, 12288)])
def test_fp8_linear_full_size_sampled(adt, M, N, K):
    """The MLP up- and down-projections of the action-DiT workload (8192 tokens,
    3072 <-> 12288); the down-projection's last wave (tiles of rows 7808 ..
    8191) runs as column blocks."""
    x, w = _inputs(M, N, K, seed=7)
    xq, sx = _quant(adt, x)
    wq, sw = _quant(adt, w)
    out32 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    adt.sage_fp8_linear(xq, sx, wq, sw, out32)
    adt.sage_check()
    rows = np.unique(np.concatenate([[0, 127, 128, 7807, 7808, M - 1], np.random.default_rng(1).choice(M, 60, replace=False),
                                     np.random.default_rng(2).choice(np.arange(7808, M), 12, replace=False)]))
    xq_h, sx_h, wq_h, sw_h = (t.cpu().numpy() for t in (xq, sx, wq, sw))
    ref = fl.fp8_linear(xq_h[rows], sx_h[rows], wq_h, sw_h)
    y = out32[torch.from_numpy(rows).cuda()].cpu().numpy()
    assert np.all(np.abs(y.astype(np.float64) - ref) <= _bound(xq_h, sx_h, wq_h, sw_h, ref, rows))
