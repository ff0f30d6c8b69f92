"""fp64 CPU oracle for non-causal multi-head attention (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports it, and it imports nothing from them: the
two share no code.  The attention arithmetic lives in ``attention_oracle.c``
(plain C, double precision, OpenMP over rows); this module compiles it with
gcc and marshals numpy arrays through ctypes.  The ragged and grouped-query
forms call the same C routine (per image, or on replicated key/value heads);
the cross-length / causal form and the prologue functions (``qkv_rope``,
``qkv_norm_rope``) are plain numpy in float64.

What it computes, per batch b and head h, on token-major ``[B, N, H, D]``
inputs (hf2q ``src/inference/vision/vit_gpu.rs``, doc of ``vit_attention_gpu``
and ``vit_attention_scores_gpu``; inferencelayer ``src/vision_gpu.rs``,
``vis_attn_coop_src`` doc, "Shape")::

    s_ij  = scale * Q[i] . K[j]
    p_ij  = softmax_j(s_ij)          (row maximum subtracted first)
    O[i]  = sum_j p_ij V[j]
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attention_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

BF16, F16, F64 = 0, 1, 2
MODE_TWO_PASS, MODE_LSE, MODE_BRUTE = 0, 1, 2

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
               "-ffp-contract=off", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        p, i64, dbl, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_double, ctypes.c_int
        lib.oracle_attention.argtypes = [p, p, p, i64, i64, i64, i64, dbl, i32, i32, p]
        lib.oracle_attention_rows.argtypes = [p, p, p, i64, i64, i64, i64, dbl, i32, i32, p, i64, p]
        lib.oracle_attention_probs.argtypes = [p, p, i64, i64, i64, i64, dbl, i32, i64, i64, p]
        lib.oracle_widen.argtypes = [p, i64, i32, p]
        for f in (lib.oracle_attention, lib.oracle_attention_rows, lib.oracle_attention_probs,
                  lib.oracle_widen, lib.oracle_num_threads):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _as_input(x: np.ndarray, dtype: int) -> np.ndarray:
    want = np.float64 if dtype == F64 else np.uint16
    x = np.ascontiguousarray(x)
    if x.dtype != want:
        raise TypeError(f"oracle input must be {want.__name__} for dtype code {dtype}, got {x.dtype}")
    return x


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def attention(q, k, v, scale: float, dtype: int, mode: int = MODE_TWO_PASS) -> np.ndarray:
    """Full output ``[B, N, H, D]`` in float64.  ``q, k, v`` are uint16 bit
    patterns (dtype BF16 or F16) or float64 arrays (dtype F64), shape [B,N,H,D]."""
    q, k, v = (_as_input(x, dtype) for x in (q, k, v))
    if q.ndim != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one [B, N, H, D] shape")
    B, N, H, D = q.shape
    out = np.empty((B, N, H, D), dtype=np.float64)
    rc = _load().oracle_attention(_ptr(q), _ptr(k), _ptr(v), B, N, H, D, float(scale), dtype, mode,
                                  _ptr(out))
    if rc:
        raise RuntimeError(f"oracle_attention failed with code {rc}")
    return out


def attention_rows(q, k, v, scale: float, dtype: int, rows, mode: int = MODE_TWO_PASS) -> np.ndarray:
    """Selected output rows: ``rows`` holds flat token-head indices
    ``(b*N + i)*H + h``; returns ``[len(rows), D]`` float64."""
    q, k, v = (_as_input(x, dtype) for x in (q, k, v))
    B, N, H, D = q.shape
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    out = np.empty((rows.size, D), dtype=np.float64)
    rc = _load().oracle_attention_rows(_ptr(q), _ptr(k), _ptr(v), B, N, H, D, float(scale), dtype,
                                       mode, _ptr(rows), rows.size, _ptr(out))
    if rc:
        raise RuntimeError(f"oracle_attention_rows failed with code {rc}")
    return out


def probs(q, k, scale: float, dtype: int, b: int, h: int) -> np.ndarray:
    """The N x N softmax probability matrix of one (b, h) slice."""
    q, k = (_as_input(x, dtype) for x in (q, k))
    B, N, H, D = q.shape
    P = np.empty((N, N), dtype=np.float64)
    rc = _load().oracle_attention_probs(_ptr(q), _ptr(k), B, N, H, D, float(scale), dtype, b, h,
                                        _ptr(P))
    if rc:
        raise RuntimeError(f"oracle_attention_probs failed with code {rc}")
    return P


def attention_ext(q, k, v, scale: float, dtype: int, causal: bool = False):
    """Attention with separate query and key lengths, an optional aligned
    causal mask, and the log-sum-exp of each row (hanzo-ml
    ``src/vulkan_backend.rs``, ``flash_attn_gpu``: ``scale`` multiplies
    Q K^T; ``causal`` lets query ``i`` attend to keys ``j <= i + (Lk - Lq)``).

    ``q``: ``[B, Lq, H, D]``, ``k``, ``v``: ``[B, Lk, H, D]`` (bit patterns of
    ``dtype``, or float64 with F64).  Returns ``(out [B, Lq, H, D],
    lse [B, H, Lq])`` in float64, ``lse = log(sum_j exp(scale * q_i . k_j))``
    over the keys the row sees.  A row that sees no key (only possible when
    Lq > Lk) gets ``out = 0`` and ``lse = -inf``.  Plain numpy, one (b, h) at
    a time: the definition written out."""
    qf, kf, vf = ((x.astype(np.float64) if dtype == F64 else widen(np.ascontiguousarray(x), dtype)) for x in (q, k, v))
    B, Lq, H, D = qf.shape
    Lk = kf.shape[1]
    out = np.zeros((B, Lq, H, D))
    lse = np.full((B, H, Lq), -np.inf)
    i = np.arange(Lq)[:, None]
    j = np.arange(Lk)[None, :]
    seen = (j <= i + (Lk - Lq)) if causal else np.ones((Lq, Lk), bool)
    rows = seen.any(axis=1)
    for b in range(B):
        for h in range(H):
            s = scale * (qf[b, :, h] @ kf[b, :, h].T)
            s = np.where(seen, s, -np.inf)
            m = np.where(rows, s.max(axis=1), 0.0)
            e = np.exp(s - m[:, None])
            tot = e.sum(axis=1)
            w = np.divide(e, tot[:, None], out=np.zeros_like(e), where=rows[:, None])
            out[b, :, h] = w @ vf[b, :, h]
            lse[b, h] = np.where(rows, m + np.log(np.where(rows, tot, 1.0)), -np.inf)
    return out, lse


def attention_gqa(q, k, v, scale: float, dtype: int, mode: int = MODE_TWO_PASS) -> np.ndarray:
    """Grouped-query attention: ``q`` is ``[B, N, H, D]``, ``k`` and ``v`` are
    ``[B, N, Hkv, D]`` with ``H`` a multiple of ``Hkv``; query head ``h``
    attends with key/value head ``h // (H // Hkv)`` (hf2q
    ``src/inference/vision/vit_gpu.rs``, doc of ``vit_repeat_kv_gpu``: each
    kv head is replicated ``num_kv_groups`` times, output row ``h`` reading
    kv head ``h / num_kv_groups``).  Written as that replication followed by
    the plain attention."""
    H, Hkv = q.shape[2], k.shape[2]
    if Hkv < 1 or H % Hkv or v.shape != k.shape or k.shape[:2] != q.shape[:2] or k.shape[3] != q.shape[3]:
        raise ValueError("k, v must be [B, N, Hkv, D] with H a multiple of Hkv")
    g = H // Hkv
    return attention(q, np.repeat(k, g, axis=2), np.repeat(v, g, axis=2), scale, dtype, mode)


def attention_varlen(q, k, v, cu_seqlens, scale: float, dtype: int, mode: int = MODE_TWO_PASS) -> np.ndarray:
    """Ragged batch of images packed along the token axis: ``q, k, v`` are
    ``[total, H, D]`` and segment s covers tokens ``cu_seqlens[s] ..
    cu_seqlens[s+1] - 1``.  Each token attends to the keys of its own segment
    only, so every segment is an independent attention problem
    (inferencelayer ``src/vision_gpu.rs``, the vision tower's ``forward``:
    attention over an image is one ragged segment given by its start
    offsets, and several images are several segments).  Returns
    ``[total, H, D]`` float64; tokens of no segment (none, for valid offsets)
    stay zero."""
    cu = [int(x) for x in cu_seqlens]
    if len(cu) < 2 or cu[0] != 0 or any(b < a for a, b in zip(cu, cu[1:])):
        raise ValueError("cu_seqlens must start at 0 and be nondecreasing")
    if cu[-1] != q.shape[0]:
        raise ValueError("cu_seqlens must end at the token count")
    out = np.zeros(q.shape, np.float64)
    for a, b in zip(cu, cu[1:]):
        if b > a:
            out[a:b] = attention(q[None, a:b], k[None, a:b], v[None, a:b], scale, dtype, mode)[0]
    return out


def attention_varlen_rows(q, k, v, cu_seqlens, scale: float, dtype: int, rows,
                          mode: int = MODE_TWO_PASS) -> np.ndarray:
    """Selected output rows of :func:`attention_varlen`: ``rows`` holds flat
    token-head indices ``i*H + h`` into ``[total, H]``; returns
    ``[len(rows), D]`` float64 in the order given.  Each row is computed
    over its own segment's keys only."""
    cu = np.asarray([int(x) for x in cu_seqlens], dtype=np.int64)
    H = q.shape[1]
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    tok = rows // H
    seg = np.searchsorted(cu, tok, side="right") - 1
    out = np.empty((rows.size, q.shape[2]), np.float64)
    for s in np.unique(seg):
        a, b = int(cu[s]), int(cu[s + 1])
        sel = np.nonzero(seg == s)[0]
        local = rows[sel] - a * H
        out[sel] = attention_rows(q[None, a:b], k[None, a:b], v[None, a:b], scale, dtype, local, mode)
    return out


def qkv_rope(qkv, cos, sin, dtype: int):
    """Split a packed QKV projection and apply the rotary embedding to q and k
    (inferencelayer ``src/vision_gpu.rs``, ``VIS_QKV_ROPE`` and its doc: the
    projection output is ``[rows, 3*hid]`` = q | k | v per token; the rope
    tables ``cos``/``sin`` are ``[rows, head_dim]`` and arrive precomputed
    (the 2-D row/column walk lives in whoever built them); element ``d`` of a
    head pairs with ``d +- head_dim/2`` through ``rotate_half``, negated on
    the low half; v is not rotated).

    ``qkv``: ``[T, 3, H, D]`` bit patterns of ``dtype`` (or float64 with
    ``dtype`` F64); ``cos``, ``sin``: ``[T, D]`` float32 (or float64).
    Returns (q, k, v) as float64 ``[T, H, D]``, unrounded::

        x'[d] = x[d] * cos[d] + rotate_half(x)[d] * sin[d]
        rotate_half(x)[d] = -x[d + D/2]  (d < D/2),   x[d - D/2]  (d >= D/2)
    """
    T, three, H, D = qkv.shape
    if three != 3 or D % 2:
        raise ValueError("qkv must be [T, 3, H, D] with D even")
    x = qkv.astype(np.float64) if dtype == F64 else widen(np.ascontiguousarray(qkv), dtype)
    c = np.asarray(cos, np.float64)[:, None, :]
    s = np.asarray(sin, np.float64)[:, None, :]
    half = D // 2

    def rope(t):
        rot = np.concatenate([-t[..., half:], t[..., :half]], axis=-1)
        return t * c + rot * s

    return rope(x[:, 0]), rope(x[:, 1]), x[:, 2].copy()


def qkv_norm_rope(qkv, cos, sin, q_norm_w, k_norm_w, eps: float, dtype: int):
    """The prologue with a per-head RMS norm of q and k ahead of the rotary
    embedding (inferencelayer ``src/vision_gpu.rs``, ``GLM_QKV_QKNORM_ROPE``
    and its doc, GLM-OCR vision tower: split the packed qkv; normalise each
    head's q row and k row over its ``head_dim`` elements by the root of
    their mean square plus ``eps``, times a per-element weight; only then
    rotate; v passes through).

    ``qkv``, ``cos``, ``sin``, ``dtype`` as in :func:`qkv_rope`;
    ``q_norm_w``, ``k_norm_w``: ``[D]`` weights (one vector for all heads);
    ``eps`` >= 0.  Returns (q, k, v) as float64 ``[T, H, D]``, unrounded::

        y[d]  = x[d] / sqrt(mean_e x[e]^2 + eps) * w[d]
        x'[d] = y[d] * cos[d] + rotate_half(y)[d] * sin[d]
    """
    T, three, H, D = qkv.shape
    if three != 3:
        raise ValueError("qkv must be [T, 3, H, D]")
    x = qkv.astype(np.float64) if dtype == F64 else widen(np.ascontiguousarray(qkv), dtype)

    def rms_norm(t, w):
        ms = np.mean(t * t, axis=-1, keepdims=True)
        return t / np.sqrt(ms + float(eps)) * np.asarray(w, np.float64)

    normed = np.stack([rms_norm(x[:, 0], q_norm_w), rms_norm(x[:, 1], k_norm_w), x[:, 2]], axis=1)
    return qkv_rope(normed, cos, sin, F64)


def widen(bits: np.ndarray, dtype: int) -> np.ndarray:
    """bf16 / f16 bit patterns to float64, exactly."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, dtype=np.float64)
    rc = _load().oracle_widen(_ptr(bits), bits.size, dtype, _ptr(out))
    if rc:
        raise RuntimeError(f"oracle_widen failed with code {rc}")
    return out


def num_threads() -> int:
    """OpenMP threads the oracle runs on."""
    return int(_load().oracle_num_threads())
