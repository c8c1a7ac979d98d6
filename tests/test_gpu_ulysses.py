"""The head-sharded (Ulysses) path with the CUDA kernels: two gloo ranks on the
one GPU of this machine.

Each rank holds a token shard [B, N/2, H, D] of a seeded global BF16 tensor
("FLUX 3 Action" (SGLang cookbook), 3.1: the multi-GPU layouts).
sp.ulysses_attention gathers its H/2 heads over all N tokens (through host
memory under gloo), runs sage_quant_qkv and sage_attn_fwd on them in the CUDA
library, and returns its token shard of the output for every head.  Each rank
checks against the single-process oracle on the whole tensor: its heads' INT8
and E4M3 codes and scales bit for bit, and its output rows (FP32) within
max-abs 2e-3 and cosine 0.9999.  The ranks' kernels never wait on each other;
only the host-side exchange joins them.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out_dir: str, B, N, H, D):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    import action_diffusion_transformers_b200 as adt
    import synth
    from action_diffusion_transformers_b200 import sp
    from oracle import sage_oracle as so

    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        qb, kb, vb = synth.generate(synth.custom(B, N, H, D, seed=23, k_sigma=4.0, v_sigma=1.0, outlier_frac=0.02))
        n, h = N // world, H // world
        tok = slice(rank * n, (rank + 1) * n)
        heads = slice(rank * h, (rank + 1) * h)
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()  # noqa: E731
        q, k, v = (dev(x[:, tok]) for x in (qb, kb, vb))
        buf = adt.Buffers(B, N, h, D, out_fp32=True)
        out = sp.ulysses_attention(q, k, v, buf)
        adt.sage_check()
        ok = {"shape": tuple(out.shape) == (B, n, H, D)}
        # this rank's heads, whole path in the oracle
        sl = (slice(None), slice(None), heads, slice(None))
        o_ref, inter = so.sage_pipeline(qb[sl], kb[sl], vb[sl])
        ok["q_codes"] = np.array_equal(buf.q_codes.cpu().numpy(), inter["q_codes"])
        ok["k_codes"] = np.array_equal(buf.k_codes.cpu().numpy(), inter["k_codes"])
        ok["v_codes"] = np.array_equal(buf.v_codes_t.cpu().numpy(), inter["v_codes_t"])
        ok["scales"] = all(np.array_equal(getattr(buf, nm).cpu().numpy().view(np.uint32), inter[nm].view(np.uint32))
                           for nm in ("q_scale", "k_scale", "v_scale", "v_mean"))
        # the returned token shard for every head against the oracle on all heads
        full, _ = so.sage_pipeline(qb, kb, vb)
        got = out.cpu().numpy().astype(np.float64)
        ref = full[:, tok].astype(np.float64)
        err = float(np.abs(got - ref).max())
        cos = float(got.ravel() @ ref.ravel() / np.sqrt((got.ravel() @ got.ravel()) * (ref.ravel() @ ref.ravel())))
        ok["max_abs"] = err <= 2e-3
        ok["cos"] = cos >= 0.9999
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(" ".join(f"{key}={int(val)}" for key, val in ok.items()) + f" err={err:.3e} cos={cos:.7f}")
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("B,N,H,D", [(1, 512, 4, 128), (2, 1024, 4, 64)])
def test_ulysses_attention_on_the_gpu(tmp_path, B, N, H, D):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path), B, N, H, D), nprocs=world, join=True,
                       start_method="spawn")
    for rank in range(world):
        res = dict(kv.split("=") for kv in open(tmp_path / f"rank{rank}.txt").read().split())
        flags = {key: val for key, val in res.items() if key not in ("err", "cos")}
        assert all(val == "1" for val in flags.values()), (rank, res)
