"""Seeded synthetic inputs shaped like the DiT attention workloads.

This module is shared by the tests and the benchmark: it feeds the same bytes
to the CUDA library and to the CPU oracle.  It holds none of the method's
arithmetic (no quantization, no attention); it only draws random numbers and
rounds them to BF16 with torch's own cast.

Workloads (token counts from the DiT pages; head count and head dim are the
stated configurations, the pages give neither):
* tiny       B=1 H=2  N=256   D=64   K offsets ~N(0, 3^2), seed 0
* action_dit B=2 H=24 N=4096  D=128  CFG cond/uncond batch of a FLUX.3 Action
                                     joint block; K offsets ~N(0, 4^2) plus 2%
                                     outlier channels x8; V offsets ~N(0, 1)
* mid_video  B=1 H=24 N=16384 D=128  distributions as action_dit
* long_video B=1 H=32 N=55296 D=128  the configuration's token count; K offsets
                                     ~N(0, 4^2); 1% heavy-tail rows, Student-t(3)
* ragged     B=1 H=24 N=20480 D=128  4 concatenated streams (text 512, video
                                     18432, video_cond 1504, action+state 32) given
                                     by cu_seqlens; full attention over the
                                     concatenation; distributions as action_dit

Recipe (one numpy PCG64 generator per call, draws in this order):
 1. Q, K, V ~ N(0, 1) float32, shape [B, N, H, D];
 2. K offset per (b, h, d) ~ N(0, k_sigma^2), added to every token;
 3. outlier channels: round(outlier_frac * D) channel indices per (b, h),
    chosen without replacement; the whole K channel (noise + offset) x 8;
 4. V offset per (b, h, d) ~ N(0, v_sigma^2) when v_sigma > 0;
 5. heavy-tail rows: for Q, K, V independently, round(heavy_frac * N) token
    indices whose every value is replaced by a Student-t(3) draw (before the
    K offset is added, so the offset stays a per-channel shift);
 6. round to BF16 (RNE) and keep the raw uint16 bit patterns.

Inputs of the fused QK RMSNorm + RoPE step (projection_outputs,
normrope_inputs): Q and K before the norm (each token vector scaled by a
log-normal factor), RMSNorm weights near 1, and the cos / sin tables of the
tokens' (t, h, w, l) positions.  The tables are built here, in float64 rounded
once to float32, because they are an input of that step (a model computes them
once per sequence layout); the step itself (norm, rotation, rounding) is not.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    N: int
    H: int
    D: int
    seed: int
    k_sigma: float = 4.0
    v_sigma: float = 1.0
    outlier_frac: float = 0.0
    heavy_frac: float = 0.0
    cu_seqlens: tuple | None = None

    @property
    def attn_ops(self) -> float:
        """INT8 QK^T plus FP8 PV multiply-adds, 2 ops each: 4 * B * H * N^2 * D."""
        return 4.0 * self.B * self.H * float(self.N) ** 2 * self.D


WORKLOADS = {
    "tiny": Workload("tiny", 1, 256, 2, 64, seed=0, k_sigma=3.0, v_sigma=0.0),
    "action_dit": Workload("action_dit", 2, 4096, 24, 128, seed=1, k_sigma=4.0,
                           v_sigma=1.0, outlier_frac=0.02),
    "mid_video": Workload("mid_video", 1, 16384, 24, 128, seed=2, k_sigma=4.0,
                          v_sigma=1.0, outlier_frac=0.02),
    "long_video": Workload("long_video", 1, 55296, 32, 128, seed=3, k_sigma=4.0,
                           v_sigma=0.0, heavy_frac=0.01),
    "ragged": Workload("ragged", 1, 20480, 24, 128, seed=4, k_sigma=4.0, v_sigma=1.0,
                       outlier_frac=0.02, cu_seqlens=(0, 512, 18944, 20448, 20480)),
}


def custom(B, N, H, D, seed, **kw) -> Workload:
    return Workload(f"custom_{B}x{N}x{H}x{D}_s{seed}", B, N, H, D, seed, **kw)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> BF16 bit patterns via torch's RNE cast."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def generate(w: Workload):
    """Return (q_bits, k_bits, v_bits), uint16 [B, N, H, D] BF16 bit patterns."""
    rng = np.random.default_rng(w.seed)
    shape = (w.B, w.N, w.H, w.D)
    q = rng.standard_normal(shape, dtype=np.float32)
    k = rng.standard_normal(shape, dtype=np.float32)
    v = rng.standard_normal(shape, dtype=np.float32)
    k_off = (rng.standard_normal((w.B, 1, w.H, w.D)) * w.k_sigma).astype(np.float32)
    n_out = int(round(w.outlier_frac * w.D))
    out_idx = []
    if n_out > 0:
        for _ in range(w.B * w.H):
            out_idx.append(rng.choice(w.D, size=n_out, replace=False))
    v_off = None
    if w.v_sigma > 0:
        v_off = (rng.standard_normal((w.B, 1, w.H, w.D)) * w.v_sigma).astype(np.float32)
    n_heavy = int(round(w.heavy_frac * w.N))
    if n_heavy > 0:
        for x in (q, k, v):
            rows = rng.choice(w.N, size=n_heavy, replace=False)
            x[:, rows] = rng.standard_t(3, size=(w.B, n_heavy, w.H, w.D)).astype(np.float32)
    k += k_off
    if n_out > 0:
        i = 0
        for b in range(w.B):
            for h in range(w.H):
                k[b, :, h, out_idx[i]] *= np.float32(8.0)
                i += 1
    if v_off is not None:
        v += v_off
    return to_bf16_bits(q), to_bf16_bits(k), to_bf16_bits(v)


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """BF16 bit patterns -> float64 values (exact widening, for FP64 references)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def sample_rows(N: int, count: int, seed: int) -> np.ndarray:
    """Seeded query rows for sampled parity: every 128-row tile's first and last
    row, all rows of a ragged last tile, and random rows up to ``count``."""
    rng = np.random.default_rng(10_000 + seed)
    fixed = set()
    for t0 in range(0, N, 128):
        fixed.add(t0)
        fixed.add(min(N, t0 + 128) - 1)
    last0 = (N // 128) * 128
    fixed.update(range(last0, N))
    fixed = sorted(fixed)
    extra = max(0, count - len(fixed))
    if extra:
        pool = np.setdiff1d(np.arange(N), np.asarray(fixed))
        if pool.size:
            fixed = sorted(set(fixed) | set(rng.choice(pool, size=min(extra, pool.size), replace=False).tolist()))
    return np.asarray(fixed, dtype=np.int64)


# ----------------------------------------------------------------------------- norm / RoPE inputs
ROPE_THETA = 10000.0


def rope_axes(D: int) -> tuple:
    """Channel pairs given to each of the four RoPE axes (t, h, w, l): D/8 each.
    The pages name the four axes but not their widths; equal widths are the
    plainest reading."""
    return (D // 8,) * 4


def rope_positions(N: int, cu_seqlens=None, grid_w: int = 32, grid_h: int = 32) -> np.ndarray:
    """Integer (t, h, w, l) positions [N, 4] of a packed joint sequence.

    Without cu_seqlens the sequence is one video latent in raster order (w
    fastest, then h, then t).  With cu_seqlens the first segment is text
    (position l = index in the segment, t = h = w = 0) and every other segment
    is a video latent of its own, in raster order from (0, 0, 0)."""
    pos = np.zeros((N, 4), dtype=np.int64)
    segs = [(0, N)] if cu_seqlens is None else list(zip(cu_seqlens[:-1], cu_seqlens[1:]))
    for s, (a, e) in enumerate(segs):
        i = np.arange(e - a)
        if cu_seqlens is not None and s == 0:
            pos[a:e, 3] = i
        else:
            pos[a:e, 0] = i // (grid_w * grid_h)
            pos[a:e, 1] = (i // grid_w) % grid_h
            pos[a:e, 2] = i % grid_w
    return pos


def rope_tables(pos: np.ndarray, D: int, theta: float = ROPE_THETA):
    """cos, sin tables (float32 [N, D/2]) of the 4-axis rotary embedding.

    Axis k owns the next rope_axes(D)[k] channel pairs; its pair j turns by
    pos[:, k] * theta ** (-j / pairs_k), formed in float64 and rounded once
    to float32 (cos and sin alike)."""
    cols = []
    for k, pairs in enumerate(rope_axes(D)):
        freq = theta ** (-np.arange(pairs, dtype=np.float64) / pairs)
        cols.append(pos[:, k:k + 1].astype(np.float64) * freq[None, :])
    ang = np.concatenate(cols, axis=1)
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def norm_weights(D: int, seed: int):
    """RMSNorm weights of Q and K: BF16 bit patterns [D], near 1 (random init)."""
    rng = np.random.default_rng(50_000 + seed)
    wq = (1.0 + 0.1 * rng.standard_normal(D)).astype(np.float32)
    wk = (1.0 + 0.1 * rng.standard_normal(D)).astype(np.float32)
    return to_bf16_bits(wq), to_bf16_bits(wk)


def normrope_inputs(w: Workload, eps: float = 1e-6) -> dict:
    """The inputs of the fused QK norm + RoPE step for a workload: weights,
    eps (binary32) and the cos / sin tables of its token positions."""
    q_w, k_w = norm_weights(w.D, w.seed)
    cos, sin = rope_tables(rope_positions(w.N, w.cu_seqlens), w.D)
    return dict(q_w=q_w, k_w=k_w, eps=float(np.float32(eps)), cos=cos, sin=sin)


def projection_outputs(w: Workload):
    """Q and K as they leave the projection (before the norm): the workload's
    Q / K with a per-token magnitude spread (log-normal, sigma 1), the scale
    that RMSNorm removes.  BF16 bit patterns [B, N, H, D]."""
    q, k, _ = generate(w)
    rng = np.random.default_rng(60_000 + w.seed)
    out = []
    for x in (q, k):
        f = bits_to_f64(x).astype(np.float32)
        f *= np.exp(rng.standard_normal((w.B, w.N, w.H, 1))).astype(np.float32)
        out.append(to_bf16_bits(f))
    return out[0], out[1]
