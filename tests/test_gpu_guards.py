"""Out-of-bounds writes: every output buffer (and the workspace) of every entry
point sits between two 4 KiB guard regions filled with a canary byte, on ragged
shapes (N not a multiple of 64 or 128, D = 64 and 128, batch 2, several
segments).  After the calls the guards must hold the canary, and the outputs
no NaN.  This stands in for a memory checker, which is not available here:
any write past a buffer's end, or before its start, changes a guard.
"""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

GUARD = 4096
CANARY = 0xA5


class Guarded:
    """A device buffer of `shape` and `dtype` between two canary-filled guards."""

    def __init__(self, shape, dtype):
        nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.nbytes = nbytes
        self.raw = torch.full((nbytes + 2 * GUARD,), CANARY, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + nbytes].view(dtype).view(shape)

    def intact(self) -> bool:
        return bool((self.raw[:GUARD] == CANARY).all()) and bool((self.raw[GUARD + self.nbytes:] == CANARY).all())


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _attention_outputs(adt, B, N, H, D, q_gran="block64", k_gran="block64"):
    Np = adt.npad(N)
    g = dict(q_codes=Guarded((B, H, Np, D), torch.int8), k_codes=Guarded((B, H, Np, D), torch.int8),
             q_scale=Guarded(adt.scale_shape(B, H, N, q_gran), torch.float32),
             k_scale=Guarded(adt.scale_shape(B, H, N, k_gran), torch.float32),
             k_mean=Guarded((B, H, D), torch.bfloat16), v_codes_t=Guarded((B, H, D, Np), torch.uint8),
             v_scale=Guarded((B, H, D), torch.float32), v_mean=Guarded((B, H, D), torch.float32))
    return g


@pytest.mark.parametrize("B,N,H,D,cu,q_gran,k_gran", [
    (1, 1, 2, 64, None, "block64", "block64"),
    (2, 65, 3, 128, None, "block64", "block64"),
    (1, 200, 2, 64, None, "token", "block64"),
    (1, 1000, 2, 128, (0, 300, 301, 1000), "segment64", "segment64"),
    (2, 1536, 2, 128, None, "block64", "token"),
])
def test_no_write_outside_the_buffers(adt, B, N, H, D, cu, q_gran, k_gran):
    w = synth.custom(B, N, H, D, seed=31, k_sigma=3.0, v_sigma=1.0)
    qb, kb, vb = synth.generate(w)
    q, k, v = _dev(qb), _dev(kb), _dev(vb)
    shape = adt.make_shape(B, N, H, D, cu_seqlens=cu, q_gran=q_gran, k_gran=k_gran)
    ws = Guarded((max(256, adt.workspace_bytes(shape)),), torch.uint8)
    g = _attention_outputs(adt, B, N, H, D, q_gran, k_gran)
    t = {name: x.t for name, x in g.items()}
    # the one-call quantization (it runs the two calls in turn for finer scale groups)
    adt.sage_quant_qkv(q, k, v, shape, 0, t["q_codes"], t["q_scale"], t["k_codes"], t["k_scale"], t["k_mean"],
                       t["v_codes_t"], t["v_scale"], t["v_mean"], ws.t)
    # the two calls on their own, into the same buffers
    adt.sage_quant_qk(q, k, shape, t["q_codes"], t["q_scale"], t["k_codes"], t["k_scale"], t["k_mean"], ws.t)
    adt.sage_quant_v(v, shape, t["v_codes_t"], t["v_scale"], t["v_mean"], ws.t)
    outs = {}
    for out_fp32 in (False, True):
        out = Guarded((B, N, H, D), torch.float32 if out_fp32 else torch.bfloat16)
        lse = Guarded((B, H, N), torch.float32)
        adt.sage_attn_fwd(t["q_codes"], t["q_scale"], t["k_codes"], t["k_scale"], t["v_codes_t"], t["v_scale"],
                          t["v_mean"], shape, 0.0, out.t, out_fp32, lse.t)
        outs[out_fp32] = (out, lse)
    adt.sage_check()
    torch.cuda.synchronize()
    for name, x in list(g.items()) + [("workspace", ws)]:
        assert x.intact(), f"a guard of {name} was overwritten"
    for out_fp32, (out, lse) in outs.items():
        assert out.intact() and lse.intact(), f"a guard of the output (fp32={out_fp32}) was overwritten"
        assert not torch.isnan(out.t.float()).any() and not torch.isnan(lse.t).any()


@pytest.mark.parametrize("B,N,H,D", [(1, 200, 2, 128), (2, 65, 2, 64)])
def test_no_write_outside_the_buffers_normrope(adt, B, N, H, D):
    w = synth.custom(B, N, H, D, seed=32, k_sigma=3.0, v_sigma=1.0)
    qb, kb = synth.projection_outputs(w)
    nr = synth.normrope_inputs(w)
    shape = adt.make_shape(B, N, H, D)
    ws = Guarded((max(256, adt.workspace_bytes(shape)),), torch.uint8)
    g = _attention_outputs(adt, B, N, H, D)
    t = {name: x.t for name, x in g.items()}
    adt.sage_quant_qk_normrope(_dev(qb), _dev(kb), shape, _dev(nr["q_w"]), _dev(nr["k_w"]),
                               torch.from_numpy(nr["cos"]).cuda(), torch.from_numpy(nr["sin"]).cuda(), nr["eps"],
                               t["q_codes"], t["q_scale"], t["k_codes"], t["k_scale"], t["k_mean"], ws.t)
    adt.sage_check()
    torch.cuda.synchronize()
    for name in ("q_codes", "q_scale", "k_codes", "k_scale", "k_mean"):
        assert g[name].intact(), f"a guard of {name} was overwritten"
    assert ws.intact()


@pytest.mark.parametrize("M,N,K", [(1, 16, 32), (200, 200, 96), (300, 1000, 4112)])
def test_no_write_outside_the_buffers_fp8_linear(adt, M, N, K):
    rng = np.random.default_rng(33)
    x = _dev(synth.to_bf16_bits(rng.standard_normal((M, K), dtype=np.float32)))
    wt = _dev(synth.to_bf16_bits(rng.standard_normal((N, K), dtype=np.float32)))
    xq, sx = Guarded((M, K), torch.uint8), Guarded((M,), torch.float32)
    wq, sw = Guarded((N, K), torch.uint8), Guarded((N,), torch.float32)
    adt.sage_fp8_quant_rows(x, xq.t, sx.t)
    adt.sage_fp8_quant_rows(wt, wq.t, sw.t)
    for dtype in (torch.bfloat16, torch.float32):
        out = Guarded((M, N), dtype)
        adt.sage_fp8_linear(xq.t, sx.t, wq.t, sw.t, out.t)
        adt.sage_check()
        torch.cuda.synchronize()
        assert out.intact(), f"a guard of the {dtype} output was overwritten"
        assert not torch.isnan(out.t.float()).any()
    for name, g in (("xq", xq), ("sx", sx), ("wq", wq), ("sw", sw)):
        assert g.intact(), f"a guard of {name} was overwritten"
