"""sage_quant_qk_static, the variant of sage_quant_qk for callers that cannot
allocate device memory (for instance a plugin whose host framework owns all
device memory, or code that must not call cudaMalloc/cudaFree because they
synchronise the device).  It keeps its scratch in a fixed array inside the
library instead of a caller workspace.

Checked through the C ABI against the existing workspace entry point: two
calls in a row on different inputs (the second smaller, so scratch left over
from the first call would show up) must give bit-identical codes, scales and
K means; and directly against the oracle (codes, scales and K means bit for
bit).  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import sage_oracle as so

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _outputs(adt, B, N, H, D):
    Np = adt.npad(N)
    return dict(q_codes=torch.full((B, H, Np, D), 7, dtype=torch.int8, device="cuda"),
                q_scale=torch.full((B, H, Np // 64), -1.0, device="cuda"),
                k_codes=torch.full((B, H, Np, D), 7, dtype=torch.int8, device="cuda"),
                k_scale=torch.full((B, H, Np // 64), -1.0, device="cuda"),
                k_mean=torch.zeros((B, H, D), dtype=torch.bfloat16, device="cuda"))


def _call(adt, fn_name, q, k, shape, o, ws=None):
    L = adt._lib
    args = [q.data_ptr(), k.data_ptr(), shape, o["q_codes"].data_ptr(), o["q_scale"].data_ptr(),
            o["k_codes"].data_ptr(), o["k_scale"].data_ptr(), o["k_mean"].data_ptr()]
    if ws is not None:
        args += [ws.data_ptr(), ws.numel()]
    args.append(torch.cuda.current_stream().cuda_stream)
    return getattr(L, fn_name)(*args)


def test_static_scratch_variant_matches_workspace_variant(adt):
    for (B, N, H, D, seed) in ((2, 2000, 6, 128, 31), (1, 333, 3, 64, 32)):
        w = synth.custom(B, N, H, D, seed=seed, k_sigma=4.0, outlier_frac=0.02)
        qb, kb, _ = synth.generate(w)
        q, k = _dev(qb), _dev(kb)
        shape = adt.make_shape(B, N, H, D)
        ref = _outputs(adt, B, N, H, D)
        ws = torch.empty(adt.workspace_bytes(shape), dtype=torch.uint8, device="cuda")
        assert _call(adt, "sage_quant_qk", q, k, shape, ref, ws) == 0
        got = _outputs(adt, B, N, H, D)
        assert _call(adt, "sage_quant_qk_static", q, k, shape, got) == 0, adt._lib.sage_last_error()
        adt.sage_check()
        for key in ref:                           # bit-exact, compared as raw bytes
            assert torch.equal(ref[key].contiguous().view(torch.uint8), got[key].contiguous().view(torch.uint8)), key
        orc = so.quant_qk(qb, kb)
        assert np.array_equal(got["q_codes"].cpu().numpy(), orc["q_codes"])
        assert np.array_equal(got["k_codes"].cpu().numpy(), orc["k_codes"])
        assert np.array_equal(got["q_scale"].cpu().numpy().view(np.uint32), orc["q_scale"].view(np.uint32))
        assert np.array_equal(got["k_scale"].cpu().numpy().view(np.uint32), orc["k_scale"].view(np.uint32))
        assert np.array_equal(got["k_mean"].cpu().view(torch.int16).numpy().view(np.uint16), orc["k_mean"])


def test_static_scratch_variant_rejects_oversized_shape(adt):
    B, N, H, D = 1, 55296, 32, 128               # needs ~28 MB of scratch
    shape = adt.make_shape(B, N, H, D)
    fake = 0x10000
    st = adt._lib.sage_quant_qk_static(fake, fake, shape, fake, fake, fake, fake, None, None)
    assert st == 6                               # SAGE_ERR_WORKSPACE, nothing launched
    assert b"scratch" in adt._lib.sage_last_error()
    adt.sage_check()
