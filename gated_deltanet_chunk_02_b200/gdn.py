"""Thin ctypes binding of libgdn (the C ABI declared in include/gdn.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors (PyTorch supplies device memory and
streams); each function passes their data pointers, the shape and the current
(or given) CUDA stream to the C entry point of the same name and raises
``GdnError`` on a nonzero return.  There is no fallback: if libgdn.so is
missing or does not load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn.so")

GDN_F32, GDN_BF16 = 0, 1
GDN_PREC_F32, GDN_PREC_F16 = 0, 1
GDN_OK, GDN_ERR_ARG, GDN_ERR_ALIGN, GDN_ERR_UNSUPPORTED, GDN_ERR_CUDA, GDN_ERR_TIMEOUT = \
    0, -1, -2, -3, -4, -5

EXPORTS = [
    "gdn_build_A", "gdn_invert_neumann", "gdn_invert_newton", "gdn_invert_blocked",
    "gdn_invert_fwdsub", "gdn_wy",
    "gdn_invert_neumann_i8", "gdn_invert_neumann_i8_residual", "gdn_invert_neumann_i16",
    "gdn_invert_neumann_i16_residual",
    "gdn_chunk_wy_fused", "gdn_chunk_wy_fused_raw", "gdn_forward",
    "gdn_forward_workspace_bytes", "gdn_forward_static", "gdn_decode", "gdn_get_status",
    "gdn_last_error", "gdn_launch_count", "gdn_debug_arm_wait_expiry", "gdn_forward_raw",
    "gdn_forward_raw_workspace_bytes",
]


class GdnShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("H", ctypes.c_int64), ("T", ctypes.c_int64),
                ("k", ctypes.c_int32), ("d", ctypes.c_int32)]


class GdnError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libgdn error {code}: {msg}")
        self.code = code


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libgdn.so (once) and declare the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise GdnError(GDN_ERR_UNSUPPORTED,
                       f"{path} is missing: build it with "
                       "`python -m gated_deltanet_chunk_02_b200.build`")
    lib = ctypes.CDLL(path)
    S = GdnShape
    sig = {
        "gdn_build_A": [_P, _P, _P, _P, S, _I, _P],
        "gdn_invert_neumann": [_P, _P, S, _I, _I, _I, _I, _P],
        "gdn_invert_newton": [_P, _P, S, _I, _I, _I, _P],
        "gdn_invert_blocked": [_P, _P, S, _P],
        "gdn_invert_fwdsub": [_P, _P, S, _P],
        "gdn_wy": [_P, _P, _P, _P, _P, _P, _P, S, _I, _P],
        "gdn_invert_neumann_i8": [_P, _P, _I, _I, _P, _P, _P, S, _P],
        "gdn_invert_neumann_i16": [_P, _P, _I, _I, _P, _P, _P, S, _P],
        "gdn_invert_neumann_i8_residual": [_P, _P, _I, _I, _I, S, _P],
        "gdn_invert_neumann_i16_residual": [_P, _P, _I, _I, _I, S, _P],
        "gdn_chunk_wy_fused": [_P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P, S, _I, _P],
        "gdn_chunk_wy_fused_raw": [_P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, S, _I,
                                   _P],
        "gdn_forward": [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _I64, S, _I, _P],
        "gdn_forward_workspace_bytes": [S, _I],
        "gdn_forward_raw": [_P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _I64, S, _I, _P],
        "gdn_forward_raw_workspace_bytes": [S, _I],
        "gdn_forward_static": [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, S, _I, _P],
        "gdn_decode": [_P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, ctypes.c_int32, _I,
                       _P],
        "gdn_get_status": [_P],
        "gdn_debug_arm_wait_expiry": [_I, _I, ctypes.c_double],
        "gdn_last_error": [],
        "gdn_launch_count": [],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = _I
    lib.gdn_forward_workspace_bytes.restype = _I64
    lib.gdn_forward_raw_workspace_bytes.restype = _I64
    lib.gdn_launch_count.restype = _I64
    lib.gdn_last_error.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _check(rc: int) -> None:
    if rc != GDN_OK:
        raise GdnError(rc, (load().gdn_last_error() or b"").decode())


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch tensor")
    if t.numel() and not t.is_cuda:
        raise ValueError("libgdn takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("libgdn takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float32:
        return GDN_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def shape(B: int, H: int, T: int, k: int, d: int = 128) -> GdnShape:
    return GdnShape(B, H, T, k, d)


def shape_of(x: torch.Tensor, k: int) -> GdnShape:
    """Shape struct of a ``[B, H, T, d]`` tensor with chunk size ``k``."""
    B, H, T, d = x.shape
    return GdnShape(B, H, T, k, d)


def shape_of_chunks(A: torch.Tensor, d: int = 128) -> GdnShape:
    """Shape struct of a ``[B, H, T/k, k, k]`` tensor (A or T)."""
    B, H, n, k, _ = A.shape
    return GdnShape(B, H, n * k, k, d)


def gdn_build_A(K, beta, g, A, k, stream=None):
    """A = -b_i (k_i . k_j) e^(g_i - g_j) below the diagonal of every chunk: K
    ``[B, H, T, d]`` (bf16 or float32), beta, g ``[B, H, T]`` float32 -> A
    ``[B, H, T/k, k, k]`` float32."""
    _check(load().gdn_build_A(_ptr(K), _ptr(beta), _ptr(g), _ptr(A), shape_of(K, k), _dtype(K),
                              _stream(stream)))


def gdn_invert_neumann(A, T, N, mask, S, prec=GDN_PREC_F32, stream=None):
    """T = truncated series of order N (band mask if ``mask``) corrected by S
    residual powers; A, T ``[B, H, T/k, k, k]`` float32; ``prec`` selects the
    fp16-operand tensor-core chain or the float32 CUDA-core one."""
    _check(load().gdn_invert_neumann(_ptr(A), _ptr(T), shape_of_chunks(A), N, int(mask), S, prec,
                                     _stream(stream)))


def gdn_invert_newton(A, T, N, mask, M, stream=None):
    """The series of order N, then M sequential corrections T <- T + T(I - (I - A)T)."""
    _check(load().gdn_invert_newton(_ptr(A), _ptr(T), shape_of_chunks(A), N, int(mask), M,
                                    _stream(stream)))


def gdn_invert_blocked(A, T, stream=None):
    """Exact T by 2 x 2 block decomposition on the tensor cores (k <= 64)."""
    _check(load().gdn_invert_blocked(_ptr(A), _ptr(T), shape_of_chunks(A), _stream(stream)))


def gdn_invert_fwdsub(A, T, stream=None):
    """Exact T by forward substitution (float32)."""
    _check(load().gdn_invert_fwdsub(_ptr(A), _ptr(T), shape_of_chunks(A), _stream(stream)))


def gdn_wy(T, K, V, beta, g, W, U, stream=None):
    """W = T diag(beta) K (W_g = T diag(beta e^g) K when ``g`` is given) and
    U = T diag(beta) V; W, U ``[B, H, T, d]`` in the dtype of K."""
    k = T.shape[-1]
    _check(load().gdn_wy(_ptr(T), _ptr(K), _ptr(V), _ptr(beta), _ptr(g), _ptr(W), _ptr(U),
                         shape_of(K, k), _dtype(K), _stream(stream)))


def gdn_invert_neumann_i8(A, T, N, mask, q=None, acc=None, scale=None, stream=None):
    """INT8 series (bit-exact scheme of gdn.h); optional dumps: codes ``q``
    int8 ``[nc, N, k, k]``, accumulators ``acc`` int32, scales float32 ``[nc, N]``."""
    _check(load().gdn_invert_neumann_i8(_ptr(A), _ptr(T), N, int(mask), _ptr(q), _ptr(acc),
                                        _ptr(scale), shape_of_chunks(A), _stream(stream)))


def gdn_invert_neumann_i8_residual(A, T, N, mask, S, stream=None):
    """INT8 series followed by S residual powers, every product in int8 codes."""
    _check(load().gdn_invert_neumann_i8_residual(_ptr(A), _ptr(T), N, int(mask), S,
                                                 shape_of_chunks(A), _stream(stream)))


def gdn_invert_neumann_i16(A, T, N, mask, q=None, acc=None, scale=None, stream=None):
    """INT16 series (int64 accumulators, binary64 scales); optional dumps: codes
    int16, accumulators int64, scales float64."""
    _check(load().gdn_invert_neumann_i16(_ptr(A), _ptr(T), N, int(mask), _ptr(q), _ptr(acc),
                                         _ptr(scale), shape_of_chunks(A), _stream(stream)))


def gdn_invert_neumann_i16_residual(A, T, N, mask, S, stream=None):
    """INT16 series followed by S residual powers, every product in int16 codes."""
    _check(load().gdn_invert_neumann_i16_residual(_ptr(A), _ptr(T), N, int(mask), S,
                                                  shape_of_chunks(A), _stream(stream)))


def gdn_chunk_wy_fused(K, V, beta, g, N, mask, S, gated, W, U, T=None, k=64, stream=None):
    """A, the series + mask + residual and W, U in one kernel; T is written
    only when a ``T`` tensor is given."""
    _check(load().gdn_chunk_wy_fused(_ptr(K), _ptr(V), _ptr(beta), _ptr(g), N, int(mask), S,
                                     int(gated), _ptr(W), _ptr(U), _ptr(T), shape_of(K, k),
                                     _dtype(K), _stream(stream)))


def gdn_chunk_wy_fused_raw(K_raw, V, beta, loggate, N, mask, S, gated, W, U, T=None,
                           K_out=None, g_out=None, k=64, stream=None):
    """The fused step from raw keys (normalised in the kernel) and per-token
    log-gates (summed chunk-locally in the kernel)."""
    _check(load().gdn_chunk_wy_fused_raw(_ptr(K_raw), _ptr(V), _ptr(beta), _ptr(loggate), N,
                                         int(mask), S, int(gated), _ptr(W), _ptr(U), _ptr(T),
                                         _ptr(K_out), _ptr(g_out), shape_of(K_raw, k),
                                         _dtype(K_raw), _stream(stream)))


def gdn_forward_workspace_bytes(K, k):
    """Scratch bytes ``gdn_forward`` needs for K's shape and dtype."""
    return int(load().gdn_forward_workspace_bytes(shape_of(K, k), _dtype(K)))


def gdn_forward(Q, K, V, beta, g, S0, N, mask, S, exact, O, S_final, workspace, k=64,
                stream=None):
    """Chunk-wise forward: O ``[B, H, T, d]`` and the final state ``S_final``
    ``[B, H, d, d]`` float32 from the start state ``S0`` (None = zero);
    ``exact`` inverts by forward substitution instead of the series."""
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().gdn_forward(_ptr(Q), _ptr(K), _ptr(V), _ptr(beta), _ptr(g), _ptr(S0), N,
                              int(mask), S, int(exact), _ptr(O), _ptr(S_final), _ptr(workspace),
                              ws, shape_of(K, k), _dtype(K), _stream(stream)))


def gdn_forward_raw_workspace_bytes(K, k):
    """Scratch bytes ``gdn_forward_raw`` needs for K's shape (bf16)."""
    return int(load().gdn_forward_raw_workspace_bytes(shape_of(K, k), _dtype(K)))


def gdn_forward_raw(Q_raw, K_raw, V, beta, loggate, S0, N, mask, S, O, S_final, workspace, k=64,
                    stream=None):
    """Chunk-wise forward from un-normalised query and key rows and per-token
    log-gates (normalised and summed in the kernels); O and the final state as
    in ``gdn_forward``."""
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().gdn_forward_raw(_ptr(Q_raw), _ptr(K_raw), _ptr(V), _ptr(beta), _ptr(loggate),
                                  _ptr(S0), N, int(mask), S, _ptr(O), _ptr(S_final),
                                  _ptr(workspace), ws, shape_of(K_raw, k), _dtype(K_raw),
                                  _stream(stream)))


def gdn_forward_static(Q, K, V, beta, g, S0, N, mask, S, exact, O, S_final, k=64, stream=None):
    """gdn_forward with the library's own fixed scratch array (no workspace, no
    allocation); see include/gdn.h for its size limit and sharing rules."""
    _check(load().gdn_forward_static(_ptr(Q), _ptr(K), _ptr(V), _ptr(beta), _ptr(g), _ptr(S0), N,
                                     int(mask), S, int(exact), _ptr(O), _ptr(S_final),
                                     shape_of(K, k), _dtype(K), _stream(stream)))


def gdn_decode(Q, K, V, beta, loggate, S, O, stream=None):
    """Decode n tokens: Q, K ``[B, Hk, n, d]``, V, O ``[B, Hv, n, d]``, beta,
    loggate ``[B, Hv, n]``, state S ``[B, Hv, d, d]`` (float32, in place)."""
    B, Hk, n, d = K.shape
    Hv = V.shape[1]
    _check(load().gdn_decode(_ptr(Q), _ptr(K), _ptr(V), _ptr(beta), _ptr(loggate), _ptr(S),
                             _ptr(O), B, Hk, Hv, n, d, _dtype(K), _stream(stream)))


def gdn_get_status(stream=None) -> int:
    """Synchronise the stream; return (and clear) the device status code."""
    return int(load().gdn_get_status(_stream(stream)))


def gdn_debug_arm_wait_expiry(tile: int, which: str, timeout_ms: float) -> None:
    """Tests only: the next fused call on this thread leaves tile ``tile``'s
    ``which`` load ("K" or "V") unissued and bounds its waits by
    ``timeout_ms`` (the wait runs out, the status word reports
    GDN_ERR_TIMEOUT)."""
    _check(load().gdn_debug_arm_wait_expiry(int(tile), {"K": 0, "V": 1}[which], float(timeout_ms)))


def gdn_last_error() -> str:
    return (load().gdn_last_error() or b"").decode()


def gdn_launch_count() -> int:
    return int(load().gdn_launch_count())
