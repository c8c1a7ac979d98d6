"""The head-sharded (Ulysses) exchange on CPU: two and four gloo ranks.

Each rank holds a token shard of a seeded global [B, N, H, D] tensor.  The
exchange must deliver exactly the global tensor's head slice (all tokens),
its inverse must give the shard back, and running the oracle's attention
path on each rank's heads, then exchanging back, must equal the
single-process oracle on the whole tensor bit for bit (the path is
independent per head).
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out_dir: str, B, N, H, D):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import synth
    from action_diffusion_transformers_b200 import sp
    from oracle import sage_oracle as so

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        qb, kb, vb = synth.generate(synth.custom(B, N, H, D, seed=21, k_sigma=3.0, v_sigma=1.0))
        n = N // world
        h = H // world
        tok = slice(rank * n, (rank + 1) * n)
        heads = slice(rank * h, (rank + 1) * h)
        as_t = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16))  # noqa: E731
        ok = {}
        shards = [as_t(x[:, tok]) for x in (qb, kb, vb)]
        gathered = [sp.seq_to_head(t) for t in shards]
        ok["gather"] = all(torch.equal(g, as_t(x[:, :, heads])) for g, x in zip(gathered, (qb, kb, vb)))
        ok["inverse"] = all(torch.equal(sp.head_to_seq(g), s) for g, s in zip(gathered, shards))
        # the whole path per rank on its heads, output exchanged back
        g_np = [g.numpy().view(np.uint16) for g in gathered]
        o_heads, _ = so.sage_pipeline(*g_np)
        o_tok = sp.head_to_seq(torch.from_numpy(np.ascontiguousarray(o_heads)))
        full, _ = so.sage_pipeline(qb, kb, vb)
        ok["attention"] = bool(np.array_equal(o_tok.numpy(), full[:, tok]))
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(" ".join(f"{k}={int(v)}" for k, v in ok.items()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,B,N,H,D", [(2, 1, 256, 4, 64), (4, 2, 512, 4, 64)])
def test_ulysses_exchange_and_attention(tmp_path, world, B, N, H, D):
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path), B, N, H, D), nprocs=world, join=True,
                       start_method="spawn")
    for rank in range(world):
        res = dict(kv.split("=") for kv in open(tmp_path / f"rank{rank}.txt").read().split())
        assert res == {"gather": "1", "inverse": "1", "attention": "1"}, (rank, res)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    from action_diffusion_transformers_b200 import sp
    x = torch.randn(1, 8, 2, 4)
    assert sp.seq_to_head(x) is x and sp.head_to_seq(x) is x


def _shape_worker(rank: int, world: int, port: int, out_dir: str):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    from action_diffusion_transformers_b200 import sp

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        res = {}
        # the checks run before any exchange, so every rank refuses alike and no collective is left waiting
        for name, fn, t in (("heads", sp.seq_to_head, torch.zeros(1, 4, 3, 8, dtype=torch.int16)),
                            ("tokens", sp.head_to_seq, torch.zeros(1, 5, 2, 8, dtype=torch.int16))):
            try:
                fn(t)
                res[name] = "accepted"
            except ValueError as e:
                res[name] = "refused" if f"{world} ranks" in str(e) else "wrong message"
        with open(os.path.join(out_dir, f"shape{rank}.txt"), "w") as f:
            f.write(" ".join(f"{k}={v}" for k, v in res.items()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_shapes_that_do_not_divide_are_refused(tmp_path):
    """H (for the gather) and N (for the return) must be multiples of the rank count."""
    mp.start_processes(_shape_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    for rank in range(2):
        res = dict(kv.split("=") for kv in open(tmp_path / f"shape{rank}.txt").read().split())
        assert res == {"heads": "refused", "tokens": "refused"}, (rank, res)
