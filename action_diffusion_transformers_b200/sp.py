"""Head-sharded (Ulysses) sequence parallelism around the quantized attention.

With P ranks, rank r holds tokens [r*N/P, (r+1)*N/P) of the joint sequence for
all H heads ([B, N/P, H, D], the sequence-parallel layout of the DiT blocks).
Every step of the attention path (K / V statistics, quantization, attention) is
independent per (b, h) and needs all N tokens of a head, so an all-to-all
brings each rank all N tokens of its H/P heads ([B, N, H/P, D]), the rank runs
the whole path on those heads with no further exchange, and a second
all-to-all returns its heads' output rows to the ranks that own the tokens.
("FLUX 3 Action" (SGLang cookbook), 3.1: the multi-GPU layouts.)

The exchange uses torch.distributed.all_to_all_single (NCCL over NVLink on
GPUs, gloo on CPU); H and N must be multiples of P.  Chunks are ordered by
rank, so the gathered token order is the global one and cu_seqlens of the
joint sequence apply unchanged.  Under gloo, device tensors are exchanged
through host memory (gloo moves host buffers); the attention itself still runs
in the CUDA kernels on each rank's GPU.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def _world(group):
    return dist.get_world_size(group) if dist.is_initialized() else 1


def _exchange(send: torch.Tensor, group) -> torch.Tensor:
    """all_to_all_single of a [P, ...] tensor, moved as bytes: 2-byte elements
    (BF16, or their int16 bit patterns) travel as int32 pairs, a type every
    backend carries."""
    if send.is_cuda and dist.get_backend(group) == "gloo":
        return _exchange(send.cpu(), group).to(send.device)
    words = send.view(torch.int32) if send.element_size() == 2 and send.shape[-1] % 2 == 0 else send
    recv = torch.empty_like(words)
    dist.all_to_all_single(recv, words, group=group)
    return recv.view(send.dtype)


def seq_to_head(x: torch.Tensor, group=None) -> torch.Tensor:
    """[B, N/P, H, D] (this rank's tokens, every head) -> [B, N, H/P, D] (every
    token, this rank's heads h in [r*H/P, (r+1)*H/P))."""
    P = _world(group)
    if P == 1:
        return x
    B, n, H, D = x.shape
    if H % P:
        raise ValueError(f"H = {H} is not a multiple of the {P} ranks")
    h = H // P
    send = x.reshape(B, n, P, h, D).permute(2, 0, 1, 3, 4).contiguous()   # chunk j: heads of rank j
    recv = _exchange(send, group)                                          # chunk s: rank s's tokens
    return recv.permute(1, 0, 2, 3, 4).reshape(B, P * n, h, D)


def head_to_seq(o: torch.Tensor, group=None) -> torch.Tensor:
    """[B, N, H/P, D] (every token, this rank's heads) -> [B, N/P, H, D] (this
    rank's tokens, every head); the inverse of seq_to_head."""
    P = _world(group)
    if P == 1:
        return o
    B, N, h, D = o.shape
    if N % P:
        raise ValueError(f"N = {N} is not a multiple of the {P} ranks")
    n = N // P
    send = o.reshape(B, P, n, h, D).permute(1, 0, 2, 3, 4).contiguous()   # chunk j: rank j's tokens
    recv = _exchange(send, group)                                          # chunk s: heads of rank s
    return recv.permute(1, 2, 0, 3, 4).reshape(B, n, P * h, D)


def ulysses_attention(q, k, v, buffers, group=None, sm_scale: float = 0.0, stream=None):
    """Quantized attention of sequence-sharded q, k, v ([B, N/P, H, D] BF16 on
    this rank's GPU).  `buffers` is a Buffers object for the gathered shape
    (B, N, H/P, D).  Returns this rank's output tokens [B, N/P, H, D]."""
    qh, kh, vh = (seq_to_head(t, group) for t in (q, k, v))
    out = buffers.run(qh, kh, vh, sm_scale=sm_scale, stream=stream)
    return head_to_seq(out, group)
