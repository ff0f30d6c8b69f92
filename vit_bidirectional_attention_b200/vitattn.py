"""Thin ctypes binding of libvitattn (the C ABI in ``include/vitattn.h``).

Argument marshalling only: every step of the attention runs in the CUDA
library.  There is no fallback: if ``libvitattn.so`` is missing this module
raises on first use, and a failing call raises :class:`VitAttnError`.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvitattn.so")

BF16, F16 = 0, 1

STATUS_NAMES = {
    0: "VITATTN_OK",
    -1: "VITATTN_ERR_NULL",
    -2: "VITATTN_ERR_DIM",
    -3: "VITATTN_ERR_HEADDIM",
    -4: "VITATTN_ERR_DTYPE",
    -5: "VITATTN_ERR_ALIGN",
    -6: "VITATTN_ERR_ALIAS",
    -7: "VITATTN_ERR_CUDA",
    -8: "VITATTN_ERR_TIMEOUT",
    -9: "VITATTN_ERR_SCALE",
    -10: "VITATTN_ERR_DEVICE",
    -11: "VITATTN_ERR_RANGE",
    -12: "VITATTN_ERR_SEQLENS",
}

_lib = None


class VitAttnError(RuntimeError):
    def __init__(self, status: int, what: str = "vitattn"):
        self.status = status
        msg = f"{what}: {STATUS_NAMES.get(status, status)} ({strerror(status)})"
        if status == -7:
            msg += f", cudaError {lib().vitattn_last_cuda_error()}"
        super().__init__(msg)


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libvitattn.so is not built ({LIB_PATH}); "
                              "run __graft_entry__.build() or vit_bidirectional_attention_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        p, i64, f32, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_int
        fwd = [p, p, p, p, i64, i64, i64, i64, f32, i32, p]
        L.vitattn_forward.argtypes = fwd
        L.vitattn_forward_checked.argtypes = fwd
        L.vitattn_test_forward_flags.argtypes = fwd + [i32]
        L.vitattn_forward_host.argtypes = [p, p, p, p, p, p, p, p, i64, i64, i64, i64, f32, i32, p]
        L.vitattn_check_args.argtypes = [p, p, p, p, i64, i64, i64, i64, f32, i32]
        var = [p, p, p, p, p, i64, i64, i64, f32, i32, p]
        L.vitattn_forward_varlen.argtypes = var
        L.vitattn_forward_varlen_checked.argtypes = var
        L.vitattn_test_forward_varlen_flags.argtypes = var + [i32]
        L.vitattn_check_args_varlen.argtypes = var[:-1]
        ext = [p, p, p, p, p, i64, i64, i64, i64, i64, f32, i32, i32, p]
        L.vitattn_forward_ext.argtypes = ext
        L.vitattn_forward_ext_checked.argtypes = ext
        L.vitattn_test_forward_ext_flags.argtypes = ext + [i32]
        L.vitattn_check_args_ext.argtypes = [p, p, p, p, p, i64, i64, i64, i64, i64, f32, i32]
        gqa = [p, p, p, p, i64, i64, i64, i64, i64, f32, i32, p]
        L.vitattn_forward_gqa.argtypes = gqa
        L.vitattn_forward_gqa_checked.argtypes = gqa
        L.vitattn_test_forward_gqa_flags.argtypes = gqa + [i32]
        L.vitattn_check_args_gqa.argtypes = gqa[:-1]
        rope = [p, p, p, p, p, p, i64, i64, i64, i32]
        L.vitattn_qkv_rope.argtypes = rope + [p]
        L.vitattn_check_args_qkv_rope.argtypes = rope
        norm_rope = [p, p, p, p, p, f32, p, p, p, i64, i64, i64, i32]
        L.vitattn_qkv_norm_rope.argtypes = norm_rope + [p]
        L.vitattn_check_args_qkv_norm_rope.argtypes = norm_rope
        strided = [p, p, p, p, i64, i64, i64, i64, i64, i64, i64, f32, i32, p]
        L.vitattn_forward_strided.argtypes = strided
        L.vitattn_forward_strided_checked.argtypes = strided
        L.vitattn_check_args_strided.argtypes = strided[:-1]
        qk_rope = [p, p, p, p, p, i64, i64, i64, i32]
        L.vitattn_qk_rope.argtypes = qk_rope + [p]
        L.vitattn_check_args_qk_rope.argtypes = qk_rope
        qk_norm_rope = [p, p, p, p, p, f32, p, p, i64, i64, i64, i32]
        L.vitattn_qk_norm_rope.argtypes = qk_norm_rope + [p]
        L.vitattn_check_args_qk_norm_rope.argtypes = qk_norm_rope
        L.vitattn_test_host_plan.argtypes = [i64, i64, i64, p]
        L.vitattn_test_host_plan.restype = ctypes.c_int
        L.vitattn_strerror.argtypes = [i32]
        L.vitattn_strerror.restype = ctypes.c_char_p
        for f in (L.vitattn_forward, L.vitattn_forward_checked, L.vitattn_test_forward_flags,
                  L.vitattn_forward_host, L.vitattn_check_args, L.vitattn_last_cuda_error,
                  L.vitattn_version, L.vitattn_launches_per_call, L.vitattn_forward_varlen,
                  L.vitattn_forward_varlen_checked, L.vitattn_test_forward_varlen_flags,
                  L.vitattn_check_args_varlen, L.vitattn_qkv_rope, L.vitattn_check_args_qkv_rope,
                  L.vitattn_forward_gqa, L.vitattn_forward_gqa_checked, L.vitattn_test_forward_gqa_flags,
                  L.vitattn_check_args_gqa, L.vitattn_forward_ext, L.vitattn_forward_ext_checked,
                  L.vitattn_test_forward_ext_flags, L.vitattn_check_args_ext, L.vitattn_qkv_norm_rope,
                  L.vitattn_check_args_qkv_norm_rope, L.vitattn_forward_strided,
                  L.vitattn_forward_strided_checked, L.vitattn_check_args_strided, L.vitattn_qk_rope,
                  L.vitattn_check_args_qk_rope, L.vitattn_qk_norm_rope, L.vitattn_check_args_qk_norm_rope):
            f.restype = ctypes.c_int
        _lib = L
    return _lib


def strerror(status: int) -> str:
    return lib().vitattn_strerror(int(status)).decode()


def version() -> int:
    return int(lib().vitattn_version())


def launches_per_call() -> int:
    return int(lib().vitattn_launches_per_call())


def host_plan(B, H, D):
    """How the host-buffer entry cuts [B, N, H, D] into copy/kernel groups:
    (images per group, groups per image -- 1 when heads are not cut, else
    part g of an image's heads is g*H//G .. (g+1)*H//G - 1 -- and groups).
    No CUDA call (a test hook of the library)."""
    out = (ctypes.c_int64 * 3)()
    rc = lib().vitattn_test_host_plan(B, H, D, ctypes.cast(out, ctypes.c_void_p))
    if rc:
        raise VitAttnError(rc)
    return tuple(int(x) for x in out)


def check_args(q, k, v, out, B, N, H, D, scale, dtype) -> int:
    """Status the library's argument checks give (pointers as ints); no CUDA call."""
    return int(lib().vitattn_check_args(q, k, v, out, B, N, H, D, float(scale), dtype))


def forward_ptr(q, k, v, out, B, N, H, D, scale, dtype, stream=0, checked=False, flags=0) -> int:
    """Raw call on device pointers (ints); returns the status code."""
    L = lib()
    args = (q, k, v, out, B, N, H, D, float(scale), dtype, stream)
    if flags:
        return int(L.vitattn_test_forward_flags(*args, int(flags)))
    if checked:
        return int(L.vitattn_forward_checked(*args))
    return int(L.vitattn_forward(*args))


def forward_host_ptr(hq, hk, hv, hout, dq, dk, dv, dout, B, N, H, D, scale, dtype, stream=0) -> int:
    """Raw host-buffer call (copies in, kernel, copy out, all enqueued on stream)."""
    return int(lib().vitattn_forward_host(hq, hk, hv, hout, dq, dk, dv, dout, B, N, H, D,
                                          float(scale), dtype, stream))


def _same_device(what: str, *tensors):
    """Raise ValueError unless every tensor lives on the first one's CUDA device.

    The call runs on that device; a tensor on another GPU would otherwise be
    read (or written) across devices by the kernel's copies."""
    dev = tensors[0].device
    for t in tensors[1:]:
        if t.device != dev:
            raise ValueError(f"{what}: every tensor must be on device {dev}, got one on {t.device}")


def _stream_handle(stream, device):
    """The raw cudaStream_t of ``stream`` (None: the device's current stream),
    refusing a torch stream of another device."""
    import torch

    if stream is None:
        stream = torch.cuda.current_stream(device)
    if isinstance(stream, int):
        return stream
    if stream.device != device:
        raise ValueError(f"stream is on {stream.device}, the tensors on {device}")
    return stream.cuda_stream


def _dtype_code(t) -> int:
    import torch

    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float16:
        return F16
    raise TypeError(f"vitattn supports bfloat16 and float16 tensors, got {t.dtype}")


def forward(q, k, v, out=None, scale=None, stream=None, checked=False):
    """O = softmax(scale * Q K^T) V per (batch, head) on CUDA tensors.

    q, k, v: contiguous ``[B, N, H, D]`` bf16 / f16 CUDA tensors (token-major,
    as a QKV linear produces them).  ``scale`` defaults to 1/sqrt(D).  Returns
    ``out`` (allocated with torch if not given).  ``checked`` synchronises and
    reports in-kernel timeouts.
    """
    import torch

    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one [B, N, H, D] shape")
    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise ValueError("q, k, v must be CUDA tensors")
    if not (q.is_contiguous() and k.is_contiguous() and v.is_contiguous()):
        raise ValueError("q, k, v must be contiguous [B, N, H, D]")
    dtype = _dtype_code(q)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype")
    B, N, H, D = q.shape
    if scale is None:
        scale = 1.0 / float(D) ** 0.5
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != q.dtype or not out.is_contiguous() or not out.is_cuda:
        raise ValueError("out must be a contiguous CUDA tensor like q")
    _same_device("vitattn_forward", q, k, v, out)
    handle = _stream_handle(stream, q.device)
    with torch.cuda.device(q.device):
        rc = forward_ptr(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, N, H, D,
                         scale, dtype, handle, checked=checked)
    if rc != 0:
        raise VitAttnError(rc, "vitattn_forward")
    return out


MAX_SEQS = 256


def _cu_array(cu_seqlens):
    """cu_seqlens as a C int32 array (host memory) and the segment count."""
    vals = [int(x) for x in cu_seqlens]
    if len(vals) < 2:
        raise ValueError("cu_seqlens needs at least two offsets")
    arr = (ctypes.c_int32 * len(vals))(*vals)
    return arr, len(vals) - 1


def check_args_varlen(q, k, v, out, cu_seqlens, H, D, scale, dtype) -> int:
    """Status the library's ragged-batch argument checks give; no CUDA call."""
    arr, n = _cu_array(cu_seqlens)
    return int(lib().vitattn_check_args_varlen(q, k, v, out, ctypes.cast(arr, ctypes.c_void_p), n, H, D,
                                               float(scale), dtype))


def forward_varlen_ptr(q, k, v, out, cu_seqlens, H, D, scale, dtype, stream=0, checked=False, flags=0) -> int:
    """Raw ragged-batch call on device pointers (ints) and host offsets; returns the status."""
    L = lib()
    arr, n = _cu_array(cu_seqlens)
    args = (q, k, v, out, ctypes.cast(arr, ctypes.c_void_p), n, H, D, float(scale), dtype, stream)
    if flags:
        return int(L.vitattn_test_forward_varlen_flags(*args, int(flags)))
    if checked:
        return int(L.vitattn_forward_varlen_checked(*args))
    return int(L.vitattn_forward_varlen(*args))


def forward_varlen(q, k, v, cu_seqlens, out=None, scale=None, stream=None, checked=False):
    """Attention within each image of a ragged batch on CUDA tensors.

    q, k, v: contiguous ``[total, H, D]`` bf16 / f16 CUDA tensors holding the
    tokens of several images back to back; ``cu_seqlens`` (a host sequence of
    ints, first 0, nondecreasing, last ``total``) gives where each image
    starts.  Every token attends only to the keys of its own image.
    ``scale`` defaults to 1/sqrt(D).  Returns ``out``.
    """
    import torch

    if q.dim() != 3 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one [total, H, D] shape")
    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise ValueError("q, k, v must be CUDA tensors")
    if not (q.is_contiguous() and k.is_contiguous() and v.is_contiguous()):
        raise ValueError("q, k, v must be contiguous [total, H, D]")
    dtype = _dtype_code(q)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype")
    if hasattr(cu_seqlens, "tolist"):
        cu_seqlens = cu_seqlens.tolist()
    total, H, D = q.shape
    if int(cu_seqlens[-1]) != total:
        raise ValueError("cu_seqlens must end at the token count")
    if scale is None:
        scale = 1.0 / float(D) ** 0.5
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != q.dtype or not out.is_contiguous() or not out.is_cuda:
        raise ValueError("out must be a contiguous CUDA tensor like q")
    _same_device("vitattn_forward_varlen", q, k, v, out)
    handle = _stream_handle(stream, q.device)
    with torch.cuda.device(q.device):
        rc = forward_varlen_ptr(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), cu_seqlens, H, D,
                                scale, dtype, handle, checked=checked)
    if rc != 0:
        raise VitAttnError(rc, "vitattn_forward_varlen")
    return out


def check_args_qkv_rope(qkv, cos, sin, q, k, v, T, H, D, dtype) -> int:
    """Status the prologue's argument checks give (pointers as ints); no CUDA call."""
    return int(lib().vitattn_check_args_qkv_rope(qkv, cos, sin, q, k, v, T, H, D, dtype))


def qkv_rope_ptr(qkv, cos, sin, q, k, v, T, H, D, dtype, stream=0) -> int:
    """Raw prologue call on device pointers (ints); returns the status."""
    return int(lib().vitattn_qkv_rope(qkv, cos, sin, q, k, v, T, H, D, dtype, stream))


def qkv_rope(qkv, cos, sin, stream=None):
    """Split a packed QKV projection and rotate q and k on CUDA tensors.

    qkv: contiguous ``[..., 3, H, D]`` bf16 / f16 (``[T, 3, H, D]`` or
    ``[B, N, 3, H, D]``); cos, sin: contiguous float32 ``[T, D]`` (one row
    per token, T = the product of the leading dims).  Returns (q, k, v), each
    ``[..., H, D]`` (the attention entries' layout).
    """
    import torch

    if qkv.dim() < 4 or qkv.shape[-3] != 3:
        raise ValueError("qkv must be [..., 3, H, D]")
    if not (qkv.is_cuda and cos.is_cuda and sin.is_cuda):
        raise ValueError("qkv, cos, sin must be CUDA tensors")
    if not (qkv.is_contiguous() and cos.is_contiguous() and sin.is_contiguous()):
        raise ValueError("qkv, cos, sin must be contiguous")
    if cos.dtype != torch.float32 or sin.dtype != torch.float32:
        raise TypeError("cos and sin must be float32")
    dtype = _dtype_code(qkv)
    lead = tuple(qkv.shape[:-3])
    H, D = qkv.shape[-2], qkv.shape[-1]
    T = 1
    for n in lead:
        T *= n
    if tuple(cos.shape) != (T, D) or tuple(sin.shape) != (T, D):
        raise ValueError("cos and sin must be [T, D] with T the token count of qkv")
    _same_device("vitattn_qkv_rope", qkv, cos, sin)
    q, k, v = (torch.empty(lead + (H, D), dtype=qkv.dtype, device=qkv.device) for _ in range(3))
    handle = _stream_handle(stream, qkv.device)
    with torch.cuda.device(qkv.device):
        rc = qkv_rope_ptr(qkv.data_ptr(), cos.data_ptr(), sin.data_ptr(), q.data_ptr(), k.data_ptr(),
                          v.data_ptr(), T, H, D, dtype, handle)
    if rc != 0:
        raise VitAttnError(rc, "vitattn_qkv_rope")
    return q, k, v


def check_args_qkv_norm_rope(qkv, cos, sin, q_norm_w, k_norm_w, eps, q, k, v, T, H, D, dtype) -> int:
    """Status the normed prologue's argument checks give (pointers as ints); no CUDA call."""
    return int(lib().vitattn_check_args_qkv_norm_rope(qkv, cos, sin, q_norm_w, k_norm_w, float(eps), q, k, v,
                                                       T, H, D, dtype))


def qkv_norm_rope_ptr(qkv, cos, sin, q_norm_w, k_norm_w, eps, q, k, v, T, H, D, dtype, stream=0) -> int:
    """Raw normed prologue call on device pointers (ints); returns the status."""
    return int(lib().vitattn_qkv_norm_rope(qkv, cos, sin, q_norm_w, k_norm_w, float(eps), q, k, v, T, H, D,
                                           dtype, stream))


def qkv_norm_rope(qkv, cos, sin, q_norm_w, k_norm_w, eps, stream=None):
    """Split a packed QKV projection, RMS-normalise each head's q and k row
    (weights ``q_norm_w``, ``k_norm_w``: contiguous float32 ``[D]`` CUDA
    tensors; ``eps`` >= 0), then rotate q and k.  Other arguments and the
    result as for :func:`qkv_rope`."""
    import torch

    if qkv.dim() < 4 or qkv.shape[-3] != 3:
        raise ValueError("qkv must be [..., 3, H, D]")
    ts = (qkv, cos, sin, q_norm_w, k_norm_w)
    if not all(t.is_cuda for t in ts):
        raise ValueError("qkv, cos, sin and the norm weights must be CUDA tensors")
    if not all(t.is_contiguous() for t in ts):
        raise ValueError("qkv, cos, sin and the norm weights must be contiguous")
    if any(t.dtype != torch.float32 for t in ts[1:]):
        raise TypeError("cos, sin and the norm weights must be float32")
    dtype = _dtype_code(qkv)
    lead = tuple(qkv.shape[:-3])
    H, D = qkv.shape[-2], qkv.shape[-1]
    T = 1
    for n in lead:
        T *= n
    if tuple(cos.shape) != (T, D) or tuple(sin.shape) != (T, D):
        raise ValueError("cos and sin must be [T, D] with T the token count of qkv")
    if tuple(q_norm_w.shape) != (D,) or tuple(k_norm_w.shape) != (D,):
        raise ValueError("the norm weights must be [D]")
    _same_device("vitattn_qkv_norm_rope", *ts)
    q, k, v = (torch.empty(lead + (H, D), dtype=qkv.dtype, device=qkv.device) for _ in range(3))
    handle = _stream_handle(stream, qkv.device)
    with torch.cuda.device(qkv.device):
        rc = qkv_norm_rope_ptr(qkv.data_ptr(), cos.data_ptr(), sin.data_ptr(), q_norm_w.data_ptr(),
                               k_norm_w.data_ptr(), eps, q.data_ptr(), k.data_ptr(), v.data_ptr(), T, H, D,
                               dtype, handle)
    if rc != 0:
        raise VitAttnError(rc, "vitattn_qkv_norm_rope")
    return q, k, v


def check_args_gqa(q, k, v, out, B, N, H, Hkv, D, scale, dtype) -> int:
    """Status the grouped-query argument checks give (pointers as ints); no CUDA call."""
    return int(lib().vitattn_check_args_gqa(q, k, v, out, B, N, H, Hkv, D, float(scale), dtype))


def forward_gqa_ptr(q, k, v, out, B, N, H, Hkv, D, scale, dtype, stream=0, checked=False, flags=0) -> int:
    """Raw grouped-query call on device pointers (ints); returns the status."""
    L = lib()
    args = (q, k, v, out, B, N, H, Hkv, D, float(scale), dtype, stream)
    if flags:
        return int(L.vitattn_test_forward_gqa_flags(*args, int(flags)))
    if checked:
        return int(L.vitattn_forward_gqa_checked(*args))
    return int(L.vitattn_forward_gqa(*args))


def forward_gqa(q, k, v, out=None, scale=None, stream=None, checked=False):
    """Grouped-query attention on CUDA tensors: q ``[B, N, H, D]``, k and v
    ``[B, N, Hkv, D]`` with H a multiple of Hkv; query head h uses key/value
    head h // (H // Hkv).  ``scale`` defaults to 1/sqrt(D).  Returns ``out``
    ``[B, N, H, D]``."""
    import torch

    if q.dim() != 4 or k.dim() != 4 or v.shape != k.shape or k.shape[:2] != q.shape[:2] or k.shape[3] != q.shape[3]:
        raise ValueError("q must be [B, N, H, D] and k, v [B, N, Hkv, D]")
    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise ValueError("q, k, v must be CUDA tensors")
    if not (q.is_contiguous() and k.is_contiguous() and v.is_contiguous()):
        raise ValueError("q, k, v must be contiguous")
    dtype = _dtype_code(q)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype")
    B, N, H, D = q.shape
    Hkv = k.shape[2]
    if scale is None:
        scale = 1.0 / float(D) ** 0.5
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != q.dtype or not out.is_contiguous() or not out.is_cuda:
        raise ValueError("out must be a contiguous CUDA tensor like q")
    _same_device("vitattn_forward_gqa", q, k, v, out)
    handle = _stream_handle(stream, q.device)
    with torch.cuda.device(q.device):
        rc = forward_gqa_ptr(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, N, H, Hkv, D, scale,
                             dtype, handle, checked=checked)
    if rc != 0:
        raise VitAttnError(rc, "vitattn_forward_gqa")
    return out


def check_args_ext(q, k, v, out, lse, B, Lq, Lk, H, D, scale, dtype) -> int:
    """Status the cross-length / causal argument checks give (pointers as ints); no CUDA call."""
    return int(lib().vitattn_check_args_ext(q, k, v, out, lse, B, Lq, Lk, H, D, float(scale), dtype))


def forward_ext_ptr(q, k, v, out, lse, B, Lq, Lk, H, D, scale, causal, dtype, stream=0, checked=False,
                    flags=0) -> int:
    """Raw cross-length / causal / LSE call on device pointers (ints; lse may be 0)."""
    L = lib()
    args = (q, k, v, out, lse or None, B, Lq, Lk, H, D, float(scale), int(bool(causal)), dtype, stream)
    if flags:
        return int(L.vitattn_test_forward_ext_flags(*args, int(flags)))
    if checked:
        return int(L.vitattn_forward_ext_checked(*args))
    return int(L.vitattn_forward_ext(*args))


def forward_ext(q, k, v, out=None, scale=None, causal=False, with_lse=False, stream=None, checked=False):
    """Attention with query length Lq and key length Lk on CUDA tensors: q
    ``[B, Lq, H, D]``, k and v ``[B, Lk, H, D]``; ``causal`` lets query i see
    keys j <= i + (Lk - Lq) only.  Returns ``out`` ``[B, Lq, H, D]``, or
    ``(out, lse)`` with ``lse`` float32 ``[B, H, Lq]`` when ``with_lse``."""
    import torch

    if q.dim() != 4 or k.dim() != 4 or v.shape != k.shape or (k.shape[0], k.shape[2], k.shape[3]) != (
            q.shape[0], q.shape[2], q.shape[3]):
        raise ValueError("q must be [B, Lq, H, D] and k, v [B, Lk, H, D]")
    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise ValueError("q, k, v must be CUDA tensors")
    if not (q.is_contiguous() and k.is_contiguous() and v.is_contiguous()):
        raise ValueError("q, k, v must be contiguous")
    dtype = _dtype_code(q)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype")
    B, Lq, H, D = q.shape
    Lk = k.shape[1]
    if scale is None:
        scale = 1.0 / float(D) ** 0.5
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != q.dtype or not out.is_contiguous() or not out.is_cuda:
        raise ValueError("out must be a contiguous CUDA tensor like q")
    _same_device("vitattn_forward_ext", q, k, v, out)
    lse = torch.empty((B, H, Lq), dtype=torch.float32, device=q.device) if with_lse else None
    handle = _stream_handle(stream, q.device)
    with torch.cuda.device(q.device):
        rc = forward_ext_ptr(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                             lse.data_ptr() if lse is not None else 0, B, Lq, Lk, H, D, scale, causal, dtype,
                             handle, checked=checked)
    if rc != 0:
        raise VitAttnError(rc, "vitattn_forward_ext")
    return (out, lse) if with_lse else out


def check_args_strided(q, k, v, out, B, N, H, D, q_stride, k_stride, v_stride, scale, dtype) -> int:
    """Status the token-strided argument checks give (pointers as ints); no CUDA call."""
    return int(lib().vitattn_check_args_strided(q, k, v, out, B, N, H, D, q_stride, k_stride, v_stride,
                                                float(scale), dtype))


def forward_strided_ptr(q, k, v, out, B, N, H, D, q_stride, k_stride, v_stride, scale, dtype, stream=0,
                        checked=False) -> int:
    """Raw token-strided call on device pointers (ints); returns the status."""
    L = lib()
    args = (q, k, v, out, B, N, H, D, q_stride, k_stride, v_stride, float(scale), dtype, stream)
    if checked:
        return int(L.vitattn_forward_strided_checked(*args))
    return int(L.vitattn_forward_strided(*args))


def _token_stride(t, N, H, D, name):
    """The element stride between tokens of a [B, N, H, D] view whose heads
    and head dims are dense (e.g. ``qkv[:, :, 0]`` of a [B, N, 3, H, D] tensor)."""
    st = t.stride()
    if st[3] != 1 or st[2] != D or st[0] != N * st[1]:
        raise ValueError(f"{name} must be a [B, N, H, D] view with dense heads and a token stride "
                         f"(strides {st})")
    return st[1]


def forward_strided(q, k, v, out=None, scale=None, stream=None, checked=False):
    """Attention on ``[B, N, H, D]`` views whose tokens need not be adjacent:
    each of q, k, v may be a column range of a packed projection, e.g.
    ``qkv.unbind(2)`` of a ``[B, N, 3, H, D]`` tensor (token stride 3*H*D),
    read in place.  ``out`` is a dense ``[B, N, H, D]`` tensor."""
    import torch

    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one [B, N, H, D] shape")
    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise ValueError("q, k, v must be CUDA tensors")
    dtype = _dtype_code(q)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype")
    B, N, H, D = q.shape
    ts = [_token_stride(t, N, H, D, n) for t, n in ((q, "q"), (k, "k"), (v, "v"))]
    if scale is None:
        scale = 1.0 / float(D) ** 0.5
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, device=q.device)
    elif out.shape != q.shape or out.dtype != q.dtype or not out.is_contiguous() or not out.is_cuda:
        raise ValueError("out must be a contiguous CUDA tensor of q's shape and dtype")
    _same_device("vitattn_forward_strided", q, k, v, out)
    handle = _stream_handle(stream, q.device)
    with torch.cuda.device(q.device):
        rc = forward_strided_ptr(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, N, H, D, *ts, scale,
                                 dtype, handle, checked=checked)
    if rc != 0:
        raise VitAttnError(rc, "vitattn_forward_strided")
    return out


def check_args_qk_rope(qkv, cos, sin, q, k, T, H, D, dtype) -> int:
    """Status the q/k-only prologue's argument checks give (pointers as ints); no CUDA call."""
    return int(lib().vitattn_check_args_qk_rope(qkv, cos, sin, q, k, T, H, D, dtype))


def qk_rope(qkv, cos, sin, q_norm_w=None, k_norm_w=None, eps=None, stream=None):
    """The prologue without the v copy: rotate q and k of a packed
    ``[..., 3, H, D]`` projection into new ``[..., H, D]`` tensors (after a
    per-head RMS norm when ``q_norm_w``, ``k_norm_w`` and ``eps`` are given)
    and return ``(q, k, v)`` with ``v`` the view ``qkv[..., 2, :, :]`` of the
    projection itself, ready for :func:`forward_strided`."""
    import torch

    if qkv.dim() < 4 or qkv.shape[-3] != 3:
        raise ValueError("qkv must be [..., 3, H, D]")
    normed = q_norm_w is not None or k_norm_w is not None or eps is not None
    ts = (qkv, cos, sin) + ((q_norm_w, k_norm_w) if normed else ())
    if normed and (q_norm_w is None or k_norm_w is None or eps is None):
        raise ValueError("the normed prologue needs q_norm_w, k_norm_w and eps")
    if not all(t.is_cuda for t in ts):
        raise ValueError("qkv, cos, sin (and the norm weights) must be CUDA tensors")
    if not all(t.is_contiguous() for t in ts):
        raise ValueError("qkv, cos, sin (and the norm weights) must be contiguous")
    if any(t.dtype != torch.float32 for t in ts[1:]):
        raise TypeError("cos, sin and the norm weights must be float32")
    dtype = _dtype_code(qkv)
    lead = tuple(qkv.shape[:-3])
    H, D = qkv.shape[-2], qkv.shape[-1]
    T = 1
    for n in lead:
        T *= n
    if tuple(cos.shape) != (T, D) or tuple(sin.shape) != (T, D):
        raise ValueError("cos and sin must be [T, D] with T the token count of qkv")
    if normed and (tuple(q_norm_w.shape) != (D,) or tuple(k_norm_w.shape) != (D,)):
        raise ValueError("the norm weights must be [D]")
    _same_device("vitattn_qk_rope", *ts)
    q, k = (torch.empty(lead + (H, D), dtype=qkv.dtype, device=qkv.device) for _ in range(2))
    handle = _stream_handle(stream, qkv.device)
    L = lib()
    with torch.cuda.device(qkv.device):
        if normed:
            rc = L.vitattn_qk_norm_rope(qkv.data_ptr(), cos.data_ptr(), sin.data_ptr(), q_norm_w.data_ptr(),
                                        k_norm_w.data_ptr(), float(eps), q.data_ptr(), k.data_ptr(), T, H, D, dtype,
                                        handle)
        else:
            rc = L.vitattn_qk_rope(qkv.data_ptr(), cos.data_ptr(), sin.data_ptr(), q.data_ptr(), k.data_ptr(), T, H,
                                   D, dtype, handle)
    if rc != 0:
        raise VitAttnError(rc, "vitattn_qk_norm_rope" if normed else "vitattn_qk_rope")
    return q, k, qkv.select(-3, 2)
