"""The whole path captured as a CUDA graph (Buffers.capture) replays the same
launches: its output equals the eager run bit for bit, also after the inputs
change in place, and a replay on new inputs matches the oracle as the eager
path does.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import sage_oracle as so

pytestmark = pytest.mark.gpu


def _dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("B,N,H,D", [(1, 300, 2, 64), (2, 512, 3, 128)])
def test_graph_replay_equals_eager_and_oracle(adt, B, N, H, D):
    w1 = synth.custom(B, N, H, D, seed=41, k_sigma=3.0, v_sigma=1.0)
    w2 = synth.custom(B, N, H, D, seed=42, k_sigma=3.0, v_sigma=1.0)
    q1, k1, v1 = synth.generate(w1)
    q2, k2, v2 = synth.generate(w2)
    q, k, v = _dev(q1), _dev(k1), _dev(v1)
    buf = adt.Buffers(B, N, H, D, out_fp32=True)
    graph = buf.capture(q, k, v)
    torch.cuda.synchronize()
    eager1 = buf.run(q, k, v).clone()
    graph.replay()
    torch.cuda.synchronize()
    adt.sage_check()
    assert torch.equal(buf.out, eager1)
    # new inputs in the captured tensors: the replay computes on them
    q.copy_(_dev(q2))
    k.copy_(_dev(k2))
    v.copy_(_dev(v2))
    graph.replay()
    torch.cuda.synchronize()
    adt.sage_check()
    replayed = buf.out.clone()
    eager2 = buf.run(q, k, v).clone()
    torch.cuda.synchronize()
    assert torch.equal(replayed, eager2)
    assert not torch.equal(replayed, eager1)
    rows = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(3).choice(N, 24, replace=False)]))
    ref, _ = so.sage_pipeline(q2, k2, v2, rows=rows)
    got = replayed.cpu().numpy()[:, rows]
    assert np.abs(got - ref).max() <= 2e-3
