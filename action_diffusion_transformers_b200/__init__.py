"""Python binding of the sm_100a quantized-attention library (libsage.so).

The three calls of the C ABI (include/sage.h) keep their names:

    sage_quant_qk(q, k, ...)   K smoothing + INT8 64-token block quantization
    sage_quant_v(v, ...)       V smoothing + per-channel E4M3, transposed
    sage_attn_fwd(...)         INT8 QK^T / FP8 PV attention, FP32 online softmax

This module only marshals arguments: torch tensors provide device memory and
the current CUDA stream; every step of the computation runs in the library's
CUDA kernels.  Importing it loads libsage.so and raises ImportError if the
library has not been built (there is no fallback implementation).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsage.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libsage.so is not built ({LIB_PATH}); run "
                      "`python -m action_diffusion_transformers_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

SAGE_OK = 0
STATUS_NAMES = {0: "SAGE_OK", 1: "SAGE_ERR_INVALID_ARG", 2: "SAGE_ERR_UNSUPPORTED", 3: "SAGE_ERR_ALIGNMENT",
                4: "SAGE_ERR_CUDA", 5: "SAGE_ERR_DEVICE_TIMEOUT", 6: "SAGE_ERR_WORKSPACE"}
EXPORTED = ("sage_npad", "sage_workspace_bytes", "sage_quant_qk", "sage_quant_v", "sage_attn_fwd",
            "sage_check", "sage_set_wait_timeout_ns", "sage_selftest_wait_timeout", "sage_last_error",
            "sage_quant_qk_static", "sage_quant_qk_normrope", "sage_fp8_quant_rows", "sage_fp8_linear",
            "sage_quant_qkv", "sage_attn_fwd_p_codes")
QK_STATIC_SCRATCH_BYTES = 8 << 20


GRAN = {"block64": 0, "token": 1, "segment64": 2}   # sage_gran: INT8 scale groups of Q / K
MAX_SEGMENTS = 256


class SageShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("N", ctypes.c_int), ("H", ctypes.c_int), ("D", ctypes.c_int),
                ("tok_stride", ctypes.c_int64), ("cu_seqlens", ctypes.POINTER(ctypes.c_int32)),
                ("n_seg", ctypes.c_int), ("q_gran", ctypes.c_int), ("k_gran", ctypes.c_int)]


class SageNormRope(ctypes.Structure):
    _fields_ = [("q_weight", ctypes.c_void_p), ("k_weight", ctypes.c_void_p), ("rope_cos", ctypes.c_void_p),
                ("rope_sin", ctypes.c_void_p), ("eps", ctypes.c_float)]


_vp = ctypes.c_void_p
_lib.sage_npad.argtypes = [ctypes.c_int]
_lib.sage_npad.restype = ctypes.c_size_t
_lib.sage_workspace_bytes.argtypes = [SageShape]
_lib.sage_workspace_bytes.restype = ctypes.c_size_t
_lib.sage_quant_qk.argtypes = [_vp, _vp, SageShape, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
_lib.sage_quant_qk.restype = ctypes.c_int
_lib.sage_quant_qk_static.argtypes = [_vp, _vp, SageShape, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.sage_quant_qk_static.restype = ctypes.c_int
_lib.sage_quant_qk_normrope.argtypes = [_vp, _vp, SageShape, ctypes.POINTER(SageNormRope), _vp, _vp, _vp, _vp, _vp,
                                        _vp, ctypes.c_size_t, _vp]
_lib.sage_quant_qk_normrope.restype = ctypes.c_int
_lib.sage_quant_qkv.argtypes = [_vp, _vp, _vp, SageShape, ctypes.c_int64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                _vp, ctypes.c_size_t, _vp]
_lib.sage_quant_qkv.restype = ctypes.c_int
_lib.sage_fp8_quant_rows.argtypes = [_vp, ctypes.c_int, ctypes.c_int, ctypes.c_int64, _vp, _vp, _vp]
_lib.sage_fp8_quant_rows.restype = ctypes.c_int
_lib.sage_fp8_linear.argtypes = [_vp, _vp, _vp, _vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp, ctypes.c_int,
                                 _vp]
_lib.sage_fp8_linear.restype = ctypes.c_int
_lib.sage_quant_v.argtypes = [_vp, SageShape, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
_lib.sage_quant_v.restype = ctypes.c_int
_lib.sage_attn_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, SageShape, ctypes.c_float, _vp, ctypes.c_int,
                               _vp, _vp]
_lib.sage_attn_fwd.restype = ctypes.c_int
_lib.sage_attn_fwd_p_codes.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, SageShape, ctypes.c_float, _vp,
                                       ctypes.c_int, _vp, _vp, _vp]
_lib.sage_attn_fwd_p_codes.restype = ctypes.c_int
_lib.sage_check.argtypes = [_vp]
_lib.sage_check.restype = ctypes.c_int
_lib.sage_set_wait_timeout_ns.argtypes = [ctypes.c_int64]
_lib.sage_set_wait_timeout_ns.restype = None
_lib.sage_selftest_wait_timeout.argtypes = [ctypes.c_int64, _vp]
_lib.sage_selftest_wait_timeout.restype = ctypes.c_int
_lib.sage_last_error.argtypes = []
_lib.sage_last_error.restype = ctypes.c_char_p


class SageError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.sage_last_error().decode(errors="replace")
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")


def _ok(status: int, where: str) -> None:
    if status != SAGE_OK:
        raise SageError(status, where)


def make_shape(B, N, H, D, tok_stride=0, cu_seqlens=None, q_gran="block64", k_gran="block64") -> SageShape:
    """q_gran / k_gran: a GRAN name (or its integer code) for the Q / K scale groups."""
    s = SageShape(B, N, H, D, int(tok_stride), None, 0, GRAN.get(q_gran, q_gran), GRAN.get(k_gran, k_gran))
    if cu_seqlens is not None:
        arr = (ctypes.c_int32 * len(cu_seqlens))(*[int(x) for x in cu_seqlens])
        s.cu_seqlens = ctypes.cast(arr, ctypes.POINTER(ctypes.c_int32))
        s.n_seg = len(cu_seqlens) - 1
        s._keep = arr  # keep the host array alive with the struct
    return s


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def npad(N: int) -> int:
    return int(_lib.sage_npad(int(N)))


def scale_shape(B: int, H: int, N: int, gran="block64") -> tuple:
    """Shape of a Q or K scale array: one per 64-token block, else one per token."""
    Np = npad(N)
    return (B, H, Np // 64) if GRAN.get(gran, gran) == GRAN["block64"] else (B, H, Np)


def workspace_bytes(shape: SageShape) -> int:
    return int(_lib.sage_workspace_bytes(shape))


def sage_quant_qk(q, k, shape, q_codes, q_scale, k_codes, k_scale, k_mean, workspace, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if hasattr(workspace, "numel") else 0
    _ok(_lib.sage_quant_qk(_ptr(q), _ptr(k), shape, _ptr(q_codes), _ptr(q_scale), _ptr(k_codes), _ptr(k_scale),
                           _ptr(k_mean), _ptr(workspace), ws_bytes, _stream(stream)), "sage_quant_qk")


def sage_quant_qk_static(q, k, shape, q_codes, q_scale, k_codes, k_scale, k_mean, stream=None):
    """sage_quant_qk without a workspace: for callers that cannot allocate
    device memory.  Scratch lives in a fixed 8 MiB array inside the library;
    larger shapes raise SageError (SAGE_ERR_WORKSPACE).  Calls that overlap on
    the GPU share that array and race."""
    _ok(_lib.sage_quant_qk_static(_ptr(q), _ptr(k), shape, _ptr(q_codes), _ptr(q_scale), _ptr(k_codes),
                                  _ptr(k_scale), _ptr(k_mean), _stream(stream)), "sage_quant_qk_static")


def sage_quant_qk_normrope(q, k, shape, q_weight, k_weight, rope_cos, rope_sin, eps, q_codes, q_scale, k_codes,
                           k_scale, k_mean, workspace, stream=None):
    """sage_quant_qk on projection outputs: QK RMSNorm (BF16 weights [D], eps)
    and RoPE (float32 cos / sin tables [N, D/2]) applied in the same kernels."""
    nr = SageNormRope(_ptr(q_weight), _ptr(k_weight), _ptr(rope_cos), _ptr(rope_sin), float(eps))
    ws_bytes = workspace.numel() * workspace.element_size() if hasattr(workspace, "numel") else 0
    _ok(_lib.sage_quant_qk_normrope(_ptr(q), _ptr(k), shape, ctypes.byref(nr), _ptr(q_codes), _ptr(q_scale),
                                    _ptr(k_codes), _ptr(k_scale), _ptr(k_mean), _ptr(workspace), ws_bytes,
                                    _stream(stream)),
        "sage_quant_qk_normrope")


def sage_quant_qkv(q, k, v, shape, v_tok_stride, q_codes, q_scale, k_codes, k_scale, k_mean, v_codes_t, v_scale,
                   v_mean, workspace, stream=None):
    """sage_quant_qk and sage_quant_v in four launches (identical outputs); v may
    have its own token stride (0 means H*D)."""
    ws_bytes = workspace.numel() * workspace.element_size() if hasattr(workspace, "numel") else 0
    _ok(_lib.sage_quant_qkv(_ptr(q), _ptr(k), _ptr(v), shape, int(v_tok_stride), _ptr(q_codes), _ptr(q_scale),
                            _ptr(k_codes), _ptr(k_scale), _ptr(k_mean), _ptr(v_codes_t), _ptr(v_scale), _ptr(v_mean),
                            _ptr(workspace), ws_bytes, _stream(stream)), "sage_quant_qkv")


def sage_fp8_quant_rows(x, codes, scale, stream=None):
    """Per-row E4M3 codes [R, K] (uint8) and scales [R] (float32) of a BF16 [R, K]
    tensor whose rows may be strided (x.stride(1) must be 1)."""
    R, K = x.shape
    assert x.stride(1) == 1
    _ok(_lib.sage_fp8_quant_rows(_ptr(x), R, K, x.stride(0), _ptr(codes), _ptr(scale), _stream(stream)),
        "sage_fp8_quant_rows")


def sage_fp8_linear(xq, sx, wq, sw, out, stream=None):
    """out [M, N] (BF16 or float32) = row-wise FP8 product of xq [M, K] and wq [N, K]."""
    M, K = xq.shape
    N = wq.shape[0]
    _ok(_lib.sage_fp8_linear(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), M, N, K, _ptr(out),
                             1 if out.dtype == torch.float32 else 0, _stream(stream)), "sage_fp8_linear")


def sage_quant_v(v, shape, v_codes_t, v_scale, v_mean, workspace, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if hasattr(workspace, "numel") else 0
    _ok(_lib.sage_quant_v(_ptr(v), shape, _ptr(v_codes_t), _ptr(v_scale), _ptr(v_mean), _ptr(workspace),
                          ws_bytes, _stream(stream)), "sage_quant_v")


def sage_attn_fwd(q_codes, q_scale, k_codes, k_scale, v_codes_t, v_scale, v_mean, shape, sm_scale, out,
                  out_fp32, lse=None, stream=None):
    _ok(_lib.sage_attn_fwd(_ptr(q_codes), _ptr(q_scale), _ptr(k_codes), _ptr(k_scale), _ptr(v_codes_t),
                           _ptr(v_scale), _ptr(v_mean), shape, float(sm_scale), _ptr(out), int(bool(out_fp32)),
                           _ptr(lse), _stream(stream)), "sage_attn_fwd")


def sage_attn_fwd_p_codes(q_codes, q_scale, k_codes, k_scale, v_codes_t, v_scale, v_mean, shape, sm_scale, out,
                          out_fp32, p_codes, lse=None, stream=None):
    """sage_attn_fwd plus the E4M3 codes of P in p_codes (uint8 [B*H, N, npad(N)]); a diagnostic."""
    _ok(_lib.sage_attn_fwd_p_codes(_ptr(q_codes), _ptr(q_scale), _ptr(k_codes), _ptr(k_scale), _ptr(v_codes_t),
                                   _ptr(v_scale), _ptr(v_mean), shape, float(sm_scale), _ptr(out),
                                   int(bool(out_fp32)), _ptr(lse), _ptr(p_codes), _stream(stream)),
        "sage_attn_fwd_p_codes")


def sage_check(stream=None) -> None:
    _ok(_lib.sage_check(_stream(stream)), "sage_check")


def sage_check_status(stream=None) -> int:
    return int(_lib.sage_check(_stream(stream)))


def set_wait_timeout_ns(ns: int) -> None:
    _lib.sage_set_wait_timeout_ns(int(ns))


def selftest_wait_timeout(timeout_ns: int, stream=None) -> None:
    _ok(_lib.sage_selftest_wait_timeout(int(timeout_ns), _stream(stream)), "sage_selftest_wait_timeout")


class Buffers:
    """Device buffers of one shape for the whole path (torch allocates them)."""

    def __init__(self, B, N, H, D, device="cuda", out_fp32=False, with_lse=False, tok_stride=0,
                 cu_seqlens=None, q_gran="block64", k_gran="block64"):
        self.shape = make_shape(B, N, H, D, tok_stride, cu_seqlens, q_gran, k_gran)
        self.B, self.N, self.H, self.D = B, N, H, D
        Np = npad(N)
        self.Npad = Np
        dev = torch.device(device)
        self.q_codes = torch.empty((B, H, Np, D), dtype=torch.int8, device=dev)
        self.k_codes = torch.empty((B, H, Np, D), dtype=torch.int8, device=dev)
        self.q_scale = torch.empty(scale_shape(B, H, N, q_gran), dtype=torch.float32, device=dev)
        self.k_scale = torch.empty(scale_shape(B, H, N, k_gran), dtype=torch.float32, device=dev)
        self.k_mean = torch.empty((B, H, D), dtype=torch.bfloat16, device=dev)
        self.v_codes_t = torch.empty((B, H, D, Np), dtype=torch.uint8, device=dev)
        self.v_scale = torch.empty((B, H, D), dtype=torch.float32, device=dev)
        self.v_mean = torch.empty((B, H, D), dtype=torch.float32, device=dev)
        self.out = torch.empty((B, N, H, D), dtype=torch.float32 if out_fp32 else torch.bfloat16, device=dev)
        self.out_fp32 = out_fp32
        self.lse = torch.empty((B, H, N), dtype=torch.float32, device=dev) if with_lse else None
        self.workspace = torch.empty(max(256, workspace_bytes(self.shape)), dtype=torch.uint8, device=dev)

    def run(self, q, k, v, sm_scale=0.0, stream=None, v_shape=None, normrope=None):
        """quant_qkv -> attn_fwd; q, k, v are BF16 [B, N, H, D] device tensors
        (v may be a token-strided view; pass v_shape with its tok_stride).  normrope:
        None, or dict(q_w, k_w, cos, sin, eps) of device tensors (and a float): Q and K
        are then projection outputs, normed and rotated inside the quantization."""
        if normrope is None:
            sage_quant_qkv(q, k, v, self.shape, (v_shape or self.shape).tok_stride, self.q_codes, self.q_scale,
                           self.k_codes, self.k_scale, self.k_mean, self.v_codes_t, self.v_scale, self.v_mean,
                           self.workspace, stream)
        else:
            nr = normrope
            sage_quant_qk_normrope(q, k, self.shape, nr["q_w"], nr["k_w"], nr["cos"], nr["sin"], nr["eps"],
                                   self.q_codes, self.q_scale, self.k_codes, self.k_scale, self.k_mean,
                                   self.workspace, stream)
            sage_quant_v(v, v_shape or self.shape, self.v_codes_t, self.v_scale, self.v_mean, self.workspace,
                         stream)
        sage_attn_fwd(self.q_codes, self.q_scale, self.k_codes, self.k_scale, self.v_codes_t, self.v_scale,
                      self.v_mean, self.shape, sm_scale, self.out, self.out_fp32, self.lse, stream)
        return self.out

    def capture(self, q, k, v, sm_scale=0.0, v_shape=None, normrope=None):
        """The launches of run() on these tensors, captured once into a CUDA
        graph; graph.replay() then re-runs them on whatever q, k, v hold, with
        less launch overhead between the kernels.  The calls run once eagerly
        first (on a side stream) so that every one-time setup happens outside
        the capture."""
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.run(q, k, v, sm_scale, side, v_shape, normrope)
        torch.cuda.current_stream().wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            self.run(q, k, v, sm_scale, side, v_shape, normrope)
        return graph
