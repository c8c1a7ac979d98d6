"""The seeded input generators follow their stated recipe (CPU only).

The workloads carry the configurations' shapes and segment layout; the draws
are deterministic per seed; K gets a per-channel offset of the stated spread
and, where asked, round(2% * D) whole channels scaled by 8 per head; V gets a
per-channel offset; heavy-tail rows replace exactly round(1% * N) token rows
of each tensor; the RoPE tables are unit rotations of the stated positions.
"""
import numpy as np
import pytest

import synth


def test_workload_table():
    w = synth.WORKLOADS
    assert (w["tiny"].B, w["tiny"].N, w["tiny"].H, w["tiny"].D) == (1, 256, 2, 64)
    assert (w["action_dit"].B, w["action_dit"].N, w["action_dit"].H, w["action_dit"].D) == (2, 4096, 24, 128)
    assert (w["mid_video"].B, w["mid_video"].N, w["mid_video"].H, w["mid_video"].D) == (1, 16384, 24, 128)
    assert (w["long_video"].B, w["long_video"].N, w["long_video"].H, w["long_video"].D) == (1, 55296, 32, 128)
    assert (w["ragged"].B, w["ragged"].N, w["ragged"].H, w["ragged"].D) == (1, 20480, 24, 128)
    assert w["ragged"].cu_seqlens == (0, 512, 18944, 20448, 20480)
    assert np.diff(w["ragged"].cu_seqlens).tolist() == [512, 18432, 1504, 32]
    assert w["action_dit"].attn_ops == 4.0 * 2 * 24 * 4096 ** 2 * 128


def test_generate_is_deterministic_and_finite_bf16():
    w = synth.custom(1, 300, 3, 64, seed=5, outlier_frac=0.02, heavy_frac=0.01)
    a = synth.generate(w)
    b = synth.generate(w)
    c = synth.generate(synth.custom(1, 300, 3, 64, seed=6, outlier_frac=0.02, heavy_frac=0.01))
    for x, y, z in zip(a, b, c):
        assert x.dtype == np.uint16 and x.shape == (1, 300, 3, 64)
        assert np.array_equal(x, y)
        assert not np.array_equal(x, z)
        assert np.all((x & 0x7F80) != 0x7F80)                  # no Inf / NaN exponent
    # the BF16 patterns are the RNE rounding of the float32 draws (Q comes first)
    plain = synth.generate(synth.custom(1, 300, 3, 64, seed=5))
    f = np.random.default_rng(5).standard_normal((1, 300, 3, 64), dtype=np.float32)
    assert np.array_equal(plain[0], synth.to_bf16_bits(f))


def test_k_offsets_and_outlier_channels():
    B, N, H, D = 2, 4096, 4, 128
    w = synth.custom(B, N, H, D, seed=7, k_sigma=4.0, v_sigma=1.0, outlier_frac=0.02)
    _, kb, vb = synth.generate(w)
    k = synth.bits_to_f64(kb)
    v = synth.bits_to_f64(vb)
    n_out = round(0.02 * D)
    assert n_out == 3
    std = k.std(axis=1)                                       # [B, H, D] spread over tokens
    means = k.mean(axis=1)
    for b in range(B):
        for h in range(H):
            big = np.sort(std[b, h])[::-1]
            assert np.all(big[:n_out] > 6.0) and np.all(big[n_out:] < 1.2)   # x8 channels vs N(0, 1) noise
    plain = std < 2.0
    # per-channel K offsets ~ N(0, 4^2): the spread of the channel means
    assert 3.4 < means[plain].std() < 4.6
    # V offsets ~ N(0, 1) per channel, V noise N(0, 1)
    assert 0.8 < v.mean(axis=1).std() < 1.2
    assert np.all(np.abs(v.std(axis=1) - 1.0) < 0.1)


def test_heavy_tail_rows_replace_whole_token_rows():
    B, N, H, D = 1, 2000, 2, 64
    base = synth.generate(synth.custom(B, N, H, D, seed=8, k_sigma=4.0, v_sigma=0.0))
    heavy = synth.generate(synth.custom(B, N, H, D, seed=8, k_sigma=4.0, v_sigma=0.0, heavy_frac=0.01))
    for x0, x1 in zip(base, heavy):
        changed = np.any(x0 != x1, axis=(0, 2, 3))
        assert changed.sum() == round(0.01 * N)               # exactly the heavy rows, per tensor
        rows = np.where(changed)[0]
        vals = synth.bits_to_f64(x1)[:, rows]
        # whole rows: every value of a replaced row differs (continuous draws)
        assert np.mean(x0[:, rows] != x1[:, rows]) > 0.99
        # Student-t(3) tails: far more |x| > 5 than the Gaussian rows
        assert np.mean(np.abs(vals - vals.mean(axis=1, keepdims=True)) > 5) > 0.005


@pytest.mark.parametrize("cu", [None, (0, 512, 18944, 20448, 20480)])
def test_rope_positions_and_tables(cu):
    N, D = 20480, 128
    pos = synth.rope_positions(N, cu)
    assert pos.shape == (N, 4)
    if cu is None:
        i = np.arange(N)
        assert np.array_equal(pos[:, 0], i // 1024) and np.array_equal(pos[:, 2], i % 32)
        assert not pos[:, 3].any()
    else:
        assert np.array_equal(pos[:512, 3], np.arange(512)) and not pos[:512, :3].any()
        for a in cu[1:-1]:
            assert not pos[a].any()                            # every video segment starts at (0, 0, 0)
        assert not pos[512:, 3].any()
    cos, sin = synth.rope_tables(pos, D)
    assert cos.shape == sin.shape == (N, D // 2) and cos.dtype == np.float32
    assert np.abs(cos.astype(np.float64) ** 2 + sin.astype(np.float64) ** 2 - 1).max() < 1e-6
    # axis 0 pair 0 turns by t radians; the last pair of axis 3 by l * 10000^(-15/16)
    assert np.allclose(cos[:, 0], np.cos(pos[:, 0]), atol=1e-7)
    assert np.allclose(sin[:, 63], np.sin(pos[:, 3] * 10000.0 ** (-15 / 16)), atol=1e-7)
