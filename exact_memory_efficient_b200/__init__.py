"""Exact memory-efficient attention for B200 (sm_100a).

Thin Python binding over the C ABI of ``libmea_attn.so`` (include/mea_attn.h).
The functions below carry the C names and only marshal arguments: tensor data
pointers, sizes and the current CUDA stream.  Every step of the computation
runs in the library's CUDA kernels; there is no CPU or PyTorch fallback, and
loading fails loudly if the library has not been built.  PyTorch is used only
to own device memory and streams.

    o, lse = attention_forward(q, k, v)                 # allocates o, lse
    dq, dk, dv = attention_backward(q, k, v, o, lse, do)  # allocates grads + workspace

k and v may have fewer heads than q (grouped- or multi-query attention); the
helpers then call the ``_gqa`` entry points.
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = [
    "MeaError", "load_library", "library_path",
    "MEA_OK", "MEA_ERR_INVALID_ARG", "MEA_ERR_UNSUPPORTED", "MEA_ERR_MISALIGNED", "MEA_ERR_WORKSPACE",
    "MEA_ERR_CUDA", "MEA_ERR_TIMEOUT", "MEA_DTYPE_F32", "MEA_DTYPE_BF16",
    "MEA_BWD_ALL", "MEA_BWD_PREPROCESS", "MEA_BWD_MAIN", "MEA_BWD_FINALIZE", "MEA_NOALLOC_SCRATCH_BYTES",
    "mea_attn_fwd", "mea_attn_bwd", "mea_attn_bwd_phase", "mea_attn_bwd_workspace_size", "mea_attn_bwd_noalloc",
    "mea_attn_bwd_accum", "mea_attn_bwd_accum_workspace_size", "mea_attn_accum_convert",
    "mea_attn_fwd_gqa", "mea_attn_bwd_gqa", "mea_attn_bwd_gqa_workspace_size", "mea_attn_fwd_fp8",
    "mea_attn_combine", "mea_attn_decode", "mea_attn_decode_workspace_size", "attention_decode",
    "mea_last_device_error",
    "mea_selftest_bounded_wait", "mea_status_string", "mea_last_error_message", "mea_version", "attention_forward", "attention_backward",
]

MEA_OK = 0
MEA_ERR_INVALID_ARG = 1
MEA_ERR_UNSUPPORTED = 2
MEA_ERR_MISALIGNED = 3
MEA_ERR_WORKSPACE = 4
MEA_ERR_CUDA = 5
MEA_ERR_TIMEOUT = 6

MEA_DTYPE_F32 = 0
MEA_DTYPE_BF16 = 1

MEA_BWD_ALL = 0
MEA_BWD_PREPROCESS = 1
MEA_BWD_MAIN = 2
MEA_BWD_FINALIZE = 3

# size of the static device scratch behind mea_attn_bwd_noalloc (include/mea_attn.h)
MEA_NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
_LIB = None


def library_path() -> str:
    return os.path.join(_PKG_DIR, "libmea_attn.so")


class MeaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        detail = mea_last_error_message()
        super().__init__(f"{where}: {mea_status_string(status)} (status {status})"
                         + (f" [{detail}]" if detail else ""))


def load_library() -> ctypes.CDLL:
    """Load libmea_attn.so from the package directory (raises if it is missing)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m exact_memory_efficient_b200.build` "
            "(there is no fallback implementation)")
    lib = ctypes.CDLL(path)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.mea_attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp]
    lib.mea_attn_fwd.restype = i
    lib.mea_attn_bwd_workspace_size.argtypes = [i, i, i, i, i, i, ctypes.POINTER(sz)]
    lib.mea_attn_bwd_workspace_size.restype = i
    lib.mea_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp, sz, vp]
    lib.mea_attn_bwd.restype = i
    lib.mea_attn_bwd_phase.argtypes = [i, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp, sz, vp]
    lib.mea_attn_bwd_phase.restype = i
    lib.mea_attn_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp]
    lib.mea_attn_bwd_noalloc.restype = i
    lib.mea_attn_bwd_accum_workspace_size.argtypes = [i, i, i, i, i, i, ctypes.POINTER(sz)]
    lib.mea_attn_bwd_accum_workspace_size.restype = i
    lib.mea_attn_bwd_accum.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp, sz, vp]
    lib.mea_attn_bwd_accum.restype = i
    lib.mea_attn_accum_convert.argtypes = [vp, vp, ctypes.c_longlong, f, i, vp]
    lib.mea_attn_accum_convert.restype = i
    lib.mea_attn_fwd_gqa.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp]
    lib.mea_attn_fwd_gqa.restype = i
    lib.mea_attn_bwd_gqa_workspace_size.argtypes = [i, i, i, i, i, i, i, ctypes.POINTER(sz)]
    lib.mea_attn_bwd_gqa_workspace_size.restype = i
    lib.mea_attn_bwd_gqa.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, sz, vp]
    lib.mea_attn_bwd_gqa.restype = i
    lib.mea_attn_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, f, f, vp]
    lib.mea_attn_fwd_fp8.restype = i
    lib.mea_attn_combine.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(vp), i, vp, vp, i, i, i, i, i, vp]
    lib.mea_attn_combine.restype = i
    lib.mea_attn_decode_workspace_size.argtypes = [i, i, i, i, i, i, i, ctypes.POINTER(sz)]
    lib.mea_attn_decode_workspace_size.restype = i
    lib.mea_attn_decode.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, sz, vp]
    lib.mea_attn_decode.restype = i
    lib.mea_selftest_bounded_wait.argtypes = [vp, vp]
    lib.mea_selftest_bounded_wait.restype = i
    lib.mea_last_device_error.argtypes = [vp]
    lib.mea_last_device_error.restype = i
    lib.mea_status_string.argtypes = [i]
    lib.mea_status_string.restype = ctypes.c_char_p
    lib.mea_last_error_message.argtypes = []
    lib.mea_last_error_message.restype = ctypes.c_char_p
    lib.mea_version.argtypes = []
    lib.mea_version.restype = i
    _LIB = lib
    return lib


def mea_status_string(status: int) -> str:
    return load_library().mea_status_string(int(status)).decode()


def mea_last_error_message() -> str:
    return load_library().mea_last_error_message().decode()


def mea_version() -> int:
    return int(load_library().mea_version())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return MEA_DTYPE_F32
    if t.dtype == torch.bfloat16:
        return MEA_DTYPE_BF16
    raise MeaError(MEA_ERR_UNSUPPORTED, f"dtype {t.dtype}")


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _check(status: int, where: str) -> None:
    if status != MEA_OK:
        raise MeaError(status, where)


def _bhnd(t: torch.Tensor, name: str):
    if t.dim() != 4:
        raise MeaError(MEA_ERR_INVALID_ARG, f"{name} must be [B, H, N, D]")
    if not t.is_contiguous():
        raise MeaError(MEA_ERR_INVALID_ARG, f"{name} must be contiguous")
    if not t.is_cuda:
        raise MeaError(MEA_ERR_INVALID_ARG, f"{name} must be a CUDA tensor")
    return t.shape


def _shape4(t, name: str):
    if t is None or t.dim() != 4:
        raise MeaError(MEA_ERR_INVALID_ARG, f"{name} must be [B, H, N, D]")
    return tuple(t.shape)


def _bwd_operands(q, k, v, o, lse, do, dq, dk, dv, where: str) -> None:
    """o, do, dq shaped like q; v, dk, dv like k; one dtype; lse fp32 [B, H, Nq]; then all
    contiguous CUDA tensors.  Checked before any launch, since the kernels index every operand
    by q's and k's sizes."""
    qs, ks = _shape4(q, "q"), _shape4(k, "k")
    for name, t, shape in (("o", o, qs), ("do", do, qs), ("dq", dq, qs), ("v", v, ks), ("dk", dk, ks),
                           ("dv", dv, ks)):
        if _shape4(t, name) != shape or t.dtype != q.dtype:
            raise MeaError(MEA_ERR_INVALID_ARG, f"{where}: {name} shape/dtype mismatch")
    if k.dtype != q.dtype:
        raise MeaError(MEA_ERR_INVALID_ARG, f"{where}: k dtype mismatch")
    if lse is None or tuple(lse.shape) != qs[:3] or lse.dtype != torch.float32:
        raise MeaError(MEA_ERR_INVALID_ARG, f"{where}: lse must be fp32 [B, H, Nq]")
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("do", do), ("dq", dq), ("dk", dk), ("dv", dv),
                    ("lse", lse)):
        if not t.is_contiguous() or not t.is_cuda:
            raise MeaError(MEA_ERR_INVALID_ARG, f"{where}: {name} must be a contiguous CUDA tensor")


def _bwd_shapes(q, k, v, o, lse, do, dq, dk, dv, where: str):
    """Shapes of a backward with one key/value head per query head: k [B, H, Nk, D] with q's B, H, D."""
    B, H, Nq, D = _shape4(q, "q")
    Bk, Hk, Nk, Dk = _shape4(k, "k")
    if (Bk, Hk, Dk) != (B, H, D):
        raise MeaError(MEA_ERR_INVALID_ARG, f"{where}: k must be [B, H, Nk, D] with q's B, H and D")
    _bwd_operands(q, k, v, o, lse, do, dq, dk, dv, where)
    return B, H, Nq, Nk, D


def mea_attn_fwd(q, k, v, o, lse, scale: float, stream=None) -> None:
    """C ``mea_attn_fwd``: writes o [B,H,Nq,D] and lse [B,H,Nq] (fp32) on the stream."""
    B, H, Nq, D = _bhnd(q, "q")
    Bk, Hk, Nk, Dk = _bhnd(k, "k")
    if (Bk, Hk, Dk) != (B, H, D) or tuple(v.shape) != tuple(k.shape) or tuple(o.shape) != tuple(q.shape):
        raise MeaError(MEA_ERR_INVALID_ARG, "mea_attn_fwd: shape mismatch")
    if tuple(lse.shape) != (B, H, Nq) or lse.dtype != torch.float32:
        raise MeaError(MEA_ERR_INVALID_ARG, "mea_attn_fwd: lse must be fp32 [B, H, Nq]")
    if not (q.dtype == k.dtype == v.dtype == o.dtype):
        raise MeaError(MEA_ERR_INVALID_ARG, "mea_attn_fwd: dtype mismatch")
    st = load_library().mea_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nq, Nk, D,
                                      float(scale), _dtype_code(q), _stream_handle(stream))
    _check(st, "mea_attn_fwd")


def mea_attn_bwd_workspace_size(B: int, H: int, Nq: int, Nk: int, D: int, dtype=torch.bfloat16) -> int:
    out = ctypes.c_size_t(0)
    code = MEA_DTYPE_BF16 if dtype == torch.bfloat16 else MEA_DTYPE_F32
    st = load_library().mea_attn_bwd_workspace_size(B, H, Nq, Nk, D, code, ctypes.byref(out))
    _check(st, "mea_attn_bwd_workspace_size")
    return int(out.value)


def mea_attn_bwd(q, k, v, o, lse, do, dq, dk, dv, scale: float, workspace, stream=None) -> None:
    """C ``mea_attn_bwd``: writes dq, dk, dv; ``workspace`` is a uint8 CUDA tensor."""
    mea_attn_bwd_phase(MEA_BWD_ALL, q, k, v, o, lse, do, dq, dk, dv, scale, workspace, stream)


def mea_attn_bwd_phase(phase: int, q, k, v, o, lse, do, dq, dk, dv, scale: float, workspace, stream=None) -> None:
    """C ``mea_attn_bwd_phase``: one phase (MEA_BWD_*) of the backward pass."""
    B, H, Nq, Nk, D = _bwd_shapes(q, k, v, o, lse, do, dq, dk, dv, "mea_attn_bwd")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load_library().mea_attn_bwd_phase(int(phase), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do),
                                            _ptr(dq), _ptr(dk), _ptr(dv), B, H, Nq, Nk, D, float(scale),
                                            _dtype_code(q), _ptr(workspace), ws_bytes, _stream_handle(stream))
    _check(st, "mea_attn_bwd_phase")


def mea_attn_bwd_noalloc(q, k, v, o, lse, do, dq, dk, dv, scale: float, stream=None) -> None:
    """C ``mea_attn_bwd_noalloc``: the backward with the library's static scratch instead of a
    caller workspace (for callers that cannot allocate; sizes up to a 64 MiB workspace)."""
    B, H, Nq, Nk, D = _bwd_shapes(q, k, v, o, lse, do, dq, dk, dv, "mea_attn_bwd_noalloc")
    st = load_library().mea_attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq),
                                              _ptr(dk), _ptr(dv), B, H, Nq, Nk, D, float(scale), _dtype_code(q),
                                              _stream_handle(stream))
    _check(st, "mea_attn_bwd_noalloc")


def mea_attn_bwd_accum_workspace_size(B: int, H: int, Nq: int, Nk: int, D: int, dtype=torch.bfloat16) -> int:
    out = ctypes.c_size_t(0)
    code = MEA_DTYPE_BF16 if dtype == torch.bfloat16 else MEA_DTYPE_F32
    st = load_library().mea_attn_bwd_accum_workspace_size(B, H, Nq, Nk, D, code, ctypes.byref(out))
    _check(st, "mea_attn_bwd_accum_workspace_size")
    return int(out.value)


def mea_attn_bwd_accum(q, k, v, o, lse, do, dq_acc, dk_acc, dv_acc, scale: float, workspace, stream=None) -> None:
    """C ``mea_attn_bwd_accum``: adds this key range's dS K, dS^T Q (both unscaled) and P^T dO to the
    fp32 sums dq_acc [B,H,Nq,D], dk_acc, dv_acc [B,H,Nk,D]; o, lse are the merged results over all keys."""
    B, H, Nq, D = _shape4(q, "q")
    Bk, Hk, Nk, Dk = _shape4(k, "k")
    if (Bk, Hk, Dk) != (B, H, D):
        raise MeaError(MEA_ERR_INVALID_ARG, "mea_attn_bwd_accum: k must be [B, H, Nk, D] with q's B, H and D")
    for name, t, shape in (("v", v, k.shape), ("o", o, q.shape), ("do", do, q.shape)):
        if tuple(t.shape) != tuple(shape) or t.dtype != q.dtype:
            raise MeaError(MEA_ERR_INVALID_ARG, f"mea_attn_bwd_accum: {name} shape/dtype mismatch")
    for name, t, shape in (("dq_acc", dq_acc, q.shape), ("dk_acc", dk_acc, k.shape), ("dv_acc", dv_acc, k.shape)):
        if tuple(t.shape) != tuple(shape) or t.dtype != torch.float32:
            raise MeaError(MEA_ERR_INVALID_ARG, f"mea_attn_bwd_accum: {name} must be fp32 shaped like q or k")
    if lse is None or tuple(lse.shape) != (B, H, Nq) or lse.dtype != torch.float32:
        raise MeaError(MEA_ERR_INVALID_ARG, "mea_attn_bwd_accum: lse must be fp32 [B, H, Nq]")
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("do", do), ("dq_acc", dq_acc), ("dk_acc", dk_acc),
                    ("dv_acc", dv_acc), ("lse", lse)):
        if not t.is_contiguous() or not t.is_cuda:
            raise MeaError(MEA_ERR_INVALID_ARG, f"mea_attn_bwd_accum: {name} must be a contiguous CUDA tensor")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load_library().mea_attn_bwd_accum(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq_acc),
                                            _ptr(dk_acc), _ptr(dv_acc), B, H, Nq, Nk, D, float(scale),
                                            _dtype_code(q), _ptr(workspace), ws_bytes, _stream_handle(stream))
    _check(st, "mea_attn_bwd_accum")


def mea_attn_accum_convert(acc, out, mul: float, stream=None) -> None:
    """C ``mea_attn_accum_convert``: out = mul * acc (fp32 sums to out's dtype, bf16 or fp32)."""
    if acc.dtype != torch.float32 or acc.shape != out.shape or not acc.is_contiguous() or not out.is_contiguous():
        raise MeaError(MEA_ERR_INVALID_ARG, "mea_attn_accum_convert: acc fp32 and out of the same shape")
    if not acc.is_cuda or not out.is_cuda:
        raise MeaError(MEA_ERR_INVALID_ARG, "mea_attn_accum_convert: CUDA tensors")
    st = load_library().mea_attn_accum_convert(_ptr(acc), _ptr(out), acc.numel(), float(mul), _dtype_code(out),
                                                _stream_handle(stream))
    _check(st, "mea_attn_accum_convert")


def _gqa_shapes(q, k, where: str, check_device: bool = True):
    B, H, Nq, D = _shape4(q, "q")
    Bk, Hkv, Nk, Dk = _shape4(k, "k")
    if (Bk, Dk) != (B, D) or Hkv < 1 or H % Hkv != 0:
        raise MeaError(MEA_ERR_INVALID_ARG, f"{where}: k must be [B, H_kv, Nk, D] with H a multiple of H_kv")
    if check_device:
        _bhnd(q, "q")
        _bhnd(k, "k")
    return B, H, Hkv, Nq, Nk, D


def mea_attn_fwd_gqa(q, k, v, o, lse, scale: float, stream=None) -> None:
    """C ``mea_attn_fwd_gqa``: q, o [B,H,Nq,D]; k, v [B,H_kv,Nk,D]; query head h reads key/value
    head h // (H // H_kv)."""
    B, H, Hkv, Nq, Nk, D = _gqa_shapes(q, k, "mea_attn_fwd_gqa")
    if tuple(v.shape) != tuple(k.shape) or tuple(o.shape) != tuple(q.shape):
        raise MeaError(MEA_ERR_INVALID_ARG, "mea_attn_fwd_gqa: shape mismatch")
    if tuple(lse.shape) != (B, H, Nq) or lse.dtype != torch.float32:
        raise MeaError(MEA_ERR_INVALID_ARG, "mea_attn_fwd_gqa: lse must be fp32 [B, H, Nq]")
    if not (q.dtype == k.dtype == v.dtype == o.dtype):
        raise MeaError(MEA_ERR_INVALID_ARG, "mea_attn_fwd_gqa: dtype mismatch")
    st = load_library().mea_attn_fwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Hkv, Nq, Nk, D,
                                          float(scale), _dtype_code(q), _stream_handle(stream))
    _check(st, "mea_attn_fwd_gqa")


def mea_attn_bwd_gqa_workspace_size(B: int, H: int, H_kv: int, Nq: int, Nk: int, D: int,
                                    dtype=torch.bfloat16) -> int:
    out = ctypes.c_size_t(0)
    code = MEA_DTYPE_BF16 if dtype == torch.bfloat16 else MEA_DTYPE_F32
    st = load_library().mea_attn_bwd_gqa_workspace_size(B, H, H_kv, Nq, Nk, D, code, ctypes.byref(out))
    _check(st, "mea_attn_bwd_gqa_workspace_size")
    return int(out.value)


def mea_attn_bwd_gqa(q, k, v, o, lse, do, dq, dk, dv, scale: float, workspace, stream=None) -> None:
    """C ``mea_attn_bwd_gqa``: dq [B,H,Nq,D]; dk, dv [B,H_kv,Nk,D] summed over each group."""
    B, H, Hkv, Nq, Nk, D = _gqa_shapes(q, k, "mea_attn_bwd_gqa", check_device=False)  # device checked below
    _bwd_operands(q, k, v, o, lse, do, dq, dk, dv, "mea_attn_bwd_gqa")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load_library().mea_attn_bwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq),
                                          _ptr(dk), _ptr(dv), B, H, Hkv, Nq, Nk, D, float(scale), _dtype_code(q),
                                          _ptr(workspace), ws_bytes, _stream_handle(stream))
    _check(st, "mea_attn_bwd_gqa")


def mea_attn_fwd_fp8(q, k, v, o, lse, scale: float, q_descale: float, k_descale: float, stream=None) -> None:
    """C ``mea_attn_fwd_fp8``: q [B,H,Nq,128] and k [B,H_kv,Nk,128] e4m3 (torch.float8_e4m3fn),
    v [B,H_kv,Nk,128] bf16; writes o [B,H,Nq,128] bf16 and lse [B,H,Nq] fp32."""
    B, H, Hkv, Nq, Nk, D = _gqa_shapes(q, k, "mea_attn_fwd_fp8")
    if q.dtype != torch.float8_e4m3fn or k.dtype != torch.float8_e4m3fn:
        raise MeaError(MEA_ERR_INVALID_ARG, "mea_attn_fwd_fp8: q and k must be float8_e4m3fn")
    if v.dtype != torch.bfloat16 or o.dtype != torch.bfloat16:
        raise MeaError(MEA_ERR_INVALID_ARG, "mea_attn_fwd_fp8: v and o must be bfloat16")
    if tuple(v.shape) != tuple(k.shape) or tuple(o.shape) != tuple(q.shape):
        raise MeaError(MEA_ERR_INVALID_ARG, "mea_attn_fwd_fp8: shape mismatch")
    if tuple(lse.shape) != (B, H, Nq) or lse.dtype != torch.float32:
        raise MeaError(MEA_ERR_INVALID_ARG, "mea_attn_fwd_fp8: lse must be fp32 [B, H, Nq]")
    st = load_library().mea_attn_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Hkv, Nq, Nk, D,
                                          float(scale), float(q_descale), float(k_descale), _stream_handle(stream))
    _check(st, "mea_attn_fwd_fp8")


def mea_attn_combine(o_parts, lse_parts, o, lse, stream=None) -> None:
    """C ``mea_attn_combine``: merge results over disjoint key ranges.  ``o_parts`` and
    ``lse_parts`` are sequences of R CUDA tensors shaped like ``o`` [B,H,Nq,D] and ``lse``
    [B,H,Nq] (fp32); writes the merged o and lse."""
    B, H, Nq, D = _bhnd(o, "o")
    R = len(o_parts)
    if R != len(lse_parts) or R < 1:
        raise MeaError(MEA_ERR_INVALID_ARG, "mea_attn_combine: one lse part per o part")
    for op, lp in zip(o_parts, lse_parts):
        if tuple(op.shape) != tuple(o.shape) or op.dtype != o.dtype or not op.is_contiguous():
            raise MeaError(MEA_ERR_INVALID_ARG, "mea_attn_combine: o parts must match o")
        if tuple(lp.shape) != (B, H, Nq) or lp.dtype != torch.float32 or not lp.is_contiguous():
            raise MeaError(MEA_ERR_INVALID_ARG, "mea_attn_combine: lse parts must be fp32 [B, H, Nq]")
    if tuple(lse.shape) != (B, H, Nq) or lse.dtype != torch.float32:
        raise MeaError(MEA_ERR_INVALID_ARG, "mea_attn_combine: lse must be fp32 [B, H, Nq]")
    optr = (ctypes.c_void_p * R)(*[_ptr(t) for t in o_parts])
    lptr = (ctypes.c_void_p * R)(*[_ptr(t) for t in lse_parts])
    st = load_library().mea_attn_combine(optr, lptr, R, _ptr(o), _ptr(lse), B, H, Nq, D, _dtype_code(o),
                                          _stream_handle(stream))
    _check(st, "mea_attn_combine")


def mea_attn_decode_workspace_size(B: int, H: int, H_kv: int, Nq: int, Nk: int, D: int,
                                   dtype=torch.bfloat16) -> int:
    """C ``mea_attn_decode_workspace_size`` (for the current CUDA device)."""
    out = ctypes.c_size_t(0)
    code = MEA_DTYPE_BF16 if dtype == torch.bfloat16 else MEA_DTYPE_F32
    st = load_library().mea_attn_decode_workspace_size(B, H, H_kv, Nq, Nk, D, code, ctypes.byref(out))
    _check(st, "mea_attn_decode_workspace_size")
    return int(out.value)


def mea_attn_decode(q, k, v, o, lse, scale: float, workspace, stream=None) -> None:
    """C ``mea_attn_decode``: the split-KV forward for few query rows per key/value head.  Shapes as
    for ``mea_attn_fwd_gqa``; ``workspace`` a CUDA tensor of at least
    ``mea_attn_decode_workspace_size`` bytes (None when that size is 0)."""
    B, H, Hkv, Nq, Nk, D = _gqa_shapes(q, k, "mea_attn_decode")
    if tuple(v.shape) != tuple(k.shape) or tuple(o.shape) != tuple(q.shape):
        raise MeaError(MEA_ERR_INVALID_ARG, "mea_attn_decode: shape mismatch")
    if tuple(lse.shape) != (B, H, Nq) or lse.dtype != torch.float32:
        raise MeaError(MEA_ERR_INVALID_ARG, "mea_attn_decode: lse must be fp32 [B, H, Nq]")
    if not (q.dtype == k.dtype == v.dtype == o.dtype):
        raise MeaError(MEA_ERR_INVALID_ARG, "mea_attn_decode: dtype mismatch")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load_library().mea_attn_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Hkv, Nq, Nk, D,
                                         float(scale), _dtype_code(q), _ptr(workspace), ws_bytes,
                                         _stream_handle(stream))
    _check(st, "mea_attn_decode")


def attention_decode(q, k, v, scale: float | None = None, stream=None):
    """Allocate (o, lse) and the workspace with torch and run ``mea_attn_decode``."""
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    B, H, Nq, D = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    n = mea_attn_decode_workspace_size(B, H, Hkv, Nq, Nk, D, q.dtype)
    ws = torch.empty(n, dtype=torch.uint8, device=q.device) if n else None
    mea_attn_decode(q, k, v, o, lse, scale, ws, stream)
    return o, lse


def mea_selftest_bounded_wait(gave_up, stream=None) -> None:
    """C ``mea_selftest_bounded_wait``: a kernel whose bounded wait must expire (about 1 s)."""
    if gave_up.dtype != torch.int32 or not gave_up.is_cuda or gave_up.numel() < 1:
        raise MeaError(MEA_ERR_INVALID_ARG, "gave_up must be an int32 CUDA tensor")
    _check(load_library().mea_selftest_bounded_wait(_ptr(gave_up), _stream_handle(stream)),
           "mea_selftest_bounded_wait")


def mea_last_device_error(stream=None) -> int:
    """C ``mea_last_device_error``: synchronises the stream and returns (and clears) the device flag."""
    return int(load_library().mea_last_device_error(_stream_handle(stream)))


# ---------------------------------------------------------------- helpers

def attention_forward(q, k, v, scale: float | None = None, stream=None):
    """Allocate (o, lse) with torch and run ``mea_attn_fwd``."""
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    if k.dim() == 4 and q.dim() == 4 and k.shape[1] != q.shape[1]:
        mea_attn_fwd_gqa(q, k, v, o, lse, scale, stream)
    else:
        mea_attn_fwd(q, k, v, o, lse, scale, stream)
    return o, lse


def attention_backward(q, k, v, o, lse, do, scale: float | None = None, workspace=None, stream=None):
    """Allocate (dq, dk, dv) and, unless given, the workspace; run ``mea_attn_bwd``."""
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    B, H, Nq, D = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if workspace is None:
        workspace = torch.empty(mea_attn_bwd_gqa_workspace_size(B, H, Hkv, Nq, Nk, D, q.dtype), dtype=torch.uint8,
                                device=q.device)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    if Hkv != H:
        mea_attn_bwd_gqa(q, k, v, o, lse, do, dq, dk, dv, scale, workspace, stream)
    else:
        mea_attn_bwd(q, k, v, o, lse, do, dq, dk, dv, scale, workspace, stream)
    return dq, dk, dv
