"""The C-ABI library on the host (no GPU needed): it loads, exports every call
declared in include/sage.h, sizes its workspace, and rejects invalid
arguments before any CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "sage.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sage_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol(adt):
    names = _declared_functions()
    assert {"sage_quant_qk", "sage_quant_v", "sage_attn_fwd"} <= set(names)
    lib = ctypes.CDLL(adt.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(adt.EXPORTED)


def test_npad_and_workspace(adt):
    assert [adt.npad(n) for n in (1, 127, 128, 129, 4096, 55296)] == [128, 128, 128, 256, 4096, 55296]
    assert adt.npad(0) == 0
    s = adt.make_shape(2, 4096, 24, 128)
    ws = adt.workspace_bytes(s)
    nsb = 4096 // 64
    assert ws >= 2 * nsb * 24 * 128 * 16 and ws % 256 == 0
    assert adt.workspace_bytes(adt.make_shape(1, 100, 2, 96)) == 0


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first or no GPU is reached


def _qk(adt, shape, **over):
    a = dict(q=FAKE, k=FAKE, qc=FAKE, qs=FAKE, kc=FAKE, ks=FAKE, km=None, ws=0x100000, wsb=1 << 40)
    a.update(over)
    return adt._lib.sage_quant_qk(a["q"], a["k"], shape, a["qc"], a["qs"], a["kc"], a["ks"], a["km"], a["ws"],
                                  a["wsb"], None)


@pytest.mark.parametrize("B,N,H,D,ts,status", [
    (1, 256, 2, 96, 0, 2),       # unsupported head dim
    (1, 0, 2, 64, 0, 1),         # empty sequence
    (0, 16, 2, 64, 0, 1),        # empty batch
    (1, 16, 2, 64, 100, 1),      # token stride below H*D
    (1, 16, 2, 64, 132, 3),      # token stride not a multiple of 8
])
def test_shape_validation(adt, B, N, H, D, ts, status):
    assert _qk(adt, adt.make_shape(B, N, H, D, ts)) == status
    assert adt._lib.sage_last_error()


def test_pointer_validation(adt):
    s = adt.make_shape(1, 256, 2, 64)
    assert _qk(adt, s, q=None) == 1
    assert _qk(adt, s, kc=FAKE + 8) == 3
    assert _qk(adt, s, km=FAKE + 2) == 3
    assert _qk(adt, s, ws=None) == 6
    assert _qk(adt, s, ws=0x100010) == 3
    assert _qk(adt, s, wsb=16) == 6
    assert b"workspace" in adt._lib.sage_last_error()


def test_cu_seqlens_validation(adt):
    ok = adt.make_shape(1, 20480, 24, 128, cu_seqlens=[0, 512, 18944, 20448, 20480])
    bad_end = adt.make_shape(1, 20480, 24, 128, cu_seqlens=[0, 512, 18944, 20448, 20479])
    bad_order = adt.make_shape(1, 20480, 24, 128, cu_seqlens=[0, 512, 400, 20480])
    bad_start = adt.make_shape(1, 20480, 24, 128, cu_seqlens=[3, 20480])
    for s in (bad_end, bad_order, bad_start):
        assert _qk(adt, s) == 1
    # valid arguments get past validation; without a GPU the device lookup fails
    # (with a GPU the fake pointers would reach a kernel, so that leg is skipped)
    if not _gpu_present():
        assert _qk(adt, ok) == 4


def _gpu_present():
    import torch
    return torch.cuda.is_available()


def test_granularity_validation(adt):
    for q_gran, k_gran in ((3, 0), (0, -1), (7, 7)):
        assert _qk(adt, adt.make_shape(1, 256, 2, 64, q_gran=q_gran, k_gran=k_gran)) == 1
        assert b"gran" in adt._lib.sage_last_error()
    many = list(range(0, 258)) + [300]                 # 258 segments
    assert _qk(adt, adt.make_shape(1, 300, 2, 64, cu_seqlens=many, k_gran="segment64")) == 2
    assert b"segments" in adt._lib.sage_last_error()
    assert _qk(adt, adt.make_shape(1, 300, 2, 64, cu_seqlens=many, q_gran="segment64")) == 2
    limit = list(range(0, 256)) + [300]                # 256 segments: accepted
    if not _gpu_present():
        assert _qk(adt, adt.make_shape(1, 300, 2, 64, cu_seqlens=limit, k_gran="segment64")) == 4
        assert _qk(adt, adt.make_shape(1, 300, 2, 64, cu_seqlens=many)) == 4   # blocks ignore the count
    assert adt.scale_shape(2, 3, 200, "block64") == (2, 3, 4)
    assert adt.scale_shape(2, 3, 200, "token") == adt.scale_shape(2, 3, 200, "segment64") == (2, 3, 256)


def test_attn_and_v_validation(adt):
    s = adt.make_shape(1, 256, 2, 64)
    L = adt._lib
    assert L.sage_attn_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, s, 0.0, None, 0, None, None) == 1
    assert L.sage_attn_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, s, float("nan"), FAKE, 0, None, None) == 1
    assert L.sage_attn_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, s, 0.0, FAKE, 0, FAKE + 2, None) == 3
    # the diagnostic form: its P-code output is required and 16-byte aligned
    assert L.sage_attn_fwd_p_codes(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, s, 0.0, FAKE, 0, None, None,
                                   None) == 1
    assert L.sage_attn_fwd_p_codes(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, s, 0.0, FAKE, 0, None, FAKE + 8,
                                   None) == 3
    assert L.sage_quant_v(FAKE, s, None, FAKE, FAKE, 0x100000, 1 << 40, None) == 1
    assert L.sage_quant_v(FAKE, adt.make_shape(1, 256, 2, 128, 200), FAKE, FAKE, FAKE, 0x100000, 1 << 40,
                          None) == 1
    assert L.sage_selftest_wait_timeout(0, None) == 1


def test_normrope_validation(adt):
    L = adt._lib
    s = adt.make_shape(1, 256, 2, 64)

    def call(nr, **over):
        a = dict(q=FAKE, k=FAKE, qc=FAKE, qs=FAKE, kc=FAKE, ks=FAKE)
        a.update(over)
        ref = ctypes.byref(nr) if nr is not None else None
        return L.sage_quant_qk_normrope(a["q"], a["k"], s, ref, a["qc"], a["qs"], a["kc"], a["ks"], None,
                                        0x100000, 1 << 40, None)

    good = dict(q_weight=FAKE, k_weight=FAKE, rope_cos=FAKE, rope_sin=FAKE, eps=1e-6)
    assert call(None) == 1
    assert call(adt.SageNormRope(**dict(good, q_weight=None))) == 1
    assert call(adt.SageNormRope(**dict(good, rope_sin=FAKE + 4))) == 3
    for eps in (0.0, -1e-6, float("inf"), float("nan")):
        assert call(adt.SageNormRope(**dict(good, eps=eps))) == 1
        assert b"eps" in L.sage_last_error()
    assert call(adt.SageNormRope(**good), q=None) == 1
    if not _gpu_present():
        assert call(adt.SageNormRope(**good)) == 4


def test_fp8_linear_validation(adt):
    L = adt._lib
    assert L.sage_fp8_quant_rows(FAKE, 4, 12, 0, FAKE, FAKE, None) == 3      # K % 8
    assert L.sage_fp8_quant_rows(FAKE, 4, 32768, 0, FAKE, FAKE, None) == 2   # K too large
    assert L.sage_fp8_quant_rows(FAKE, 4, 64, 60, FAKE, FAKE, None) == 3     # ld < K
    assert L.sage_fp8_quant_rows(None, 4, 64, 0, FAKE, FAKE, None) == 1
    assert L.sage_fp8_linear(FAKE, FAKE, FAKE, FAKE, 16, 16, 24, FAKE, 0, None) == 3   # K % 16
    assert L.sage_fp8_linear(FAKE, FAKE, FAKE, FAKE, 16, 12, 32, FAKE, 0, None) == 3   # N % 8
    assert L.sage_fp8_linear(FAKE, FAKE, FAKE, FAKE, 0, 16, 32, FAKE, 0, None) == 1
    assert L.sage_fp8_linear(FAKE, FAKE, FAKE + 4, FAKE, 16, 16, 32, FAKE, 0, None) == 3
    if not _gpu_present():
        assert L.sage_fp8_linear(FAKE, FAKE, FAKE, FAKE, 16, 16, 32, FAKE, 0, None) == 4


def _qkv(adt, shape, **over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, vts=0, qc=FAKE, qs=FAKE, kc=FAKE, ks=FAKE, km=None, vc=FAKE, vs=FAKE, vm=FAKE,
             ws=0x100000, wsb=1 << 40)
    a.update(over)
    return adt._lib.sage_quant_qkv(a["q"], a["k"], a["v"], shape, a["vts"], a["qc"], a["qs"], a["kc"], a["ks"],
                                   a["km"], a["vc"], a["vs"], a["vm"], a["ws"], a["wsb"], None)


def test_quant_qkv_validation(adt):
    """The one-call quantization checks its shape, V's token stride, every
    pointer and the workspace before any CUDA call."""
    assert _qkv(adt, adt.make_shape(1, 256, 2, 96)) == 2          # unsupported head dim
    assert _qkv(adt, adt.make_shape(1, 0, 2, 64)) == 1            # empty sequence
    s = adt.make_shape(1, 256, 2, 64)
    assert _qkv(adt, s, vts=100) == 1                             # V token stride below H*D
    assert _qkv(adt, s, vts=132) == 3                             # V token stride not a multiple of 8
    for name in ("q", "k", "v", "qc", "qs", "kc", "ks", "vc", "vs", "vm"):
        assert _qkv(adt, s, **{name: None}) == 1, name
    assert _qkv(adt, s, km=FAKE + 2) == 3                         # k_mean alignment
    assert _qkv(adt, s, ws=None) == 6
    assert _qkv(adt, s, wsb=16) == 6
    assert b"workspace" in adt._lib.sage_last_error()
    if not _gpu_present():
        assert _qkv(adt, s) == 4                                  # valid: stops at the device lookup
        assert _qkv(adt, s, vts=256) == 4                         # a strided V view is valid too


def test_quant_qk_static_validation(adt):
    """The allocation-free variant validates like sage_quant_qk and refuses
    shapes whose scratch exceeds its built-in array."""
    lib = adt._lib
    s = adt.make_shape(1, 256, 2, 64)
    args = [FAKE, FAKE, s, FAKE, FAKE, FAKE, FAKE, None, None]
    assert lib.sage_quant_qk_static(*args[:2], adt.make_shape(1, 256, 2, 96), *args[3:]) == 2
    for i in (0, 1, 3, 4, 5, 6):
        bad = list(args)
        bad[i] = None
        assert lib.sage_quant_qk_static(*bad) == 1, i
    bad = list(args)
    bad[7] = FAKE + 2
    assert lib.sage_quant_qk_static(*bad) == 3
    big = adt.make_shape(2, 55296, 32, 128)                       # FP64 partial sums far above 8 MiB
    assert lib.sage_quant_qk_static(FAKE, FAKE, big, FAKE, FAKE, FAKE, FAKE, None, None) == 6
    assert b"scratch" in lib.sage_last_error()


def test_selftest_timeout_range(adt):
    """The bounded-wait self-test accepts only timeouts in (0, 10 s]."""
    for bad in (0, -5, 10_000_000_001):
        assert adt._lib.sage_selftest_wait_timeout(bad, None) == 1
        assert b"timeout" in adt._lib.sage_last_error()
