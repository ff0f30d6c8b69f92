"""The C ABI without a GPU: the library loads, exports every symbol the header
declares, and its argument checks return the documented codes before any
CUDA call (hanzo-ml ``src/vulkan_backend.rs``, ``flash_attn_gpu``: sizes are
checked before dispatch; hf2q ``src/inference/vision/vit_gpu.rs``,
``vit_attention_scores_gpu`` "# Errors": zero dims are rejected)."""
import os
import re
import subprocess

import numpy as np
import pytest

from vit_bidirectional_attention_b200 import vitattn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vitattn.h")

A = 1 << 20  # fake, 16-byte aligned "device" addresses: nothing is dereferenced
BYTES = 1 * 64 * 2 * 64 * 2
Q, K, V, O = A, A + 4 * BYTES, A + 8 * BYTES, A + 12 * BYTES


def header_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"VITATTN_API\s+[\w\s\*]*?\b(vitattn_\w+)\s*\(", text)))


def test_library_loads_and_exports_every_declared_symbol():
    names = header_functions()
    assert "vitattn_forward" in names and len(names) >= 8
    L = vitattn.lib()
    for n in names:
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", vitattn.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (vitattn_\w+)", out))
    assert set(names) <= exported


def test_header_enum_values_match_binding():
    text = open(HEADER).read()
    for name, val in re.findall(r"(VITATTN_(?:OK|ERR_\w+))\s*=\s*(-?\d+)", text):
        assert vitattn.STATUS_NAMES[int(val)] == name
    assert re.search(r"VITATTN_BF16\s*=\s*0", text) and re.search(r"VITATTN_F16\s*=\s*1", text)


def test_version_and_launch_count():
    assert vitattn.version() == 10000
    assert vitattn.launches_per_call() == 1


def ok_args(**kw):
    a = dict(q=Q, k=K, v=V, out=O, B=1, N=64, H=2, D=64, scale=0.125, dtype=vitattn.BF16)
    a.update(kw)
    return a


def check(**kw):
    a = ok_args(**kw)
    return vitattn.check_args(a["q"], a["k"], a["v"], a["out"], a["B"], a["N"], a["H"], a["D"],
                              a["scale"], a["dtype"])


def test_valid_arguments_pass():
    assert check() == 0
    for D in (16, 24, 64, 72, 80, 128):
        assert check(D=D) == 0, D
    assert check(dtype=vitattn.F16, scale=-2.0) == 0
    assert check(scale=0.0) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), -1), (dict(k=0), -1), (dict(v=0), -1), (dict(out=0), -1),
    (dict(B=0), -2), (dict(N=0), -2), (dict(H=0), -2), (dict(N=-5), -2),
    (dict(N=2**31), -2), (dict(B=2**40), -2),
    (dict(D=8), -3), (dict(D=136), -3), (dict(D=70), -3), (dict(D=0), -2),
    (dict(dtype=2), -4), (dict(dtype=-1), -4),
    (dict(q=Q + 8), -5), (dict(out=O + 2), -5),
    (dict(out=Q), -6), (dict(out=K + 16), -6), (dict(out=V - 16), -6),
    (dict(scale=float("nan")), -9), (dict(scale=float("inf")), -9),
])
def test_argument_errors(kw, code):
    assert check(**kw) == code
    assert vitattn.strerror(code) not in ("ok", "unknown status")


def test_forward_rejects_bad_arguments_before_any_cuda_call():
    # these return from the checks, so they are safe on a machine without a GPU
    assert vitattn.forward_ptr(0, K, V, O, 1, 64, 2, 64, 0.125, 0) == -1
    assert vitattn.forward_ptr(Q, K, V, O, 1, 64, 2, 60, 0.125, 0) == -3
    assert vitattn.forward_ptr(Q, K, V, Q, 1, 64, 2, 64, 0.125, 0) == -6
    assert vitattn.forward_host_ptr(0, 1, 1, 1, Q, K, V, O, 1, 64, 2, 64, 0.125, 0) == -1


def test_strerror_unknown():
    assert vitattn.strerror(12345) == "unknown status"


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(vitattn, "_lib", None)
    monkeypatch.setattr(vitattn, "LIB_PATH", "/nonexistent/libvitattn.so")
    with pytest.raises(ImportError):
        vitattn.lib()


# ---------------------------------------------------------------- ragged batches

def check_var(cu=(0, 40, 64), **kw):
    a = dict(q=Q, k=K, v=V, out=O, H=2, D=64, scale=0.125, dtype=vitattn.BF16)
    a.update(kw)
    return vitattn.check_args_varlen(a["q"], a["k"], a["v"], a["out"], list(cu), a["H"], a["D"], a["scale"],
                                     a["dtype"])


def test_varlen_valid_arguments_pass():
    assert check_var() == 0
    assert check_var(cu=(0, 0, 64)) == 0            # empty segments are allowed
    assert check_var(cu=(0, 64)) == 0
    assert check_var(cu=[0] + [1] * 255 + [2], D=16) == 0  # 256 segments
    assert check_var(D=128, dtype=vitattn.F16) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), -1), (dict(out=0), -1),
    (dict(cu=(1, 40, 64)), -12), (dict(cu=(0, 40, 30)), -12), (dict(cu=(0, -1, 5)), -12),
    (dict(cu=[0] * 258), -2), (dict(H=0), -2), (dict(cu=(0, 2**31 - 1)), -2),
    (dict(D=60), -3), (dict(dtype=3), -4), (dict(q=Q + 4), -5),
    (dict(out=K + 32), -6), (dict(scale=float("nan")), -9),
])
def test_varlen_argument_errors(kw, code):
    assert check_var(**kw) == code
    assert vitattn.strerror(code) not in ("ok", "unknown status")


def test_varlen_with_no_tokens_is_a_no_op_without_cuda():
    assert vitattn.forward_varlen_ptr(Q, K, V, O, [0, 0, 0], 2, 64, 0.125, vitattn.BF16) == 0
    assert vitattn.forward_varlen_ptr(Q, K, V, O, [0, 5, 3], 2, 64, 0.125, vitattn.BF16) == -12


# ---------------------------------------------------------------- QKV split + rope prologue

def check_rope(**kw):
    T, H, D = kw.get("T", 64), kw.get("H", 2), kw.get("D", 64)
    row = max(H * D * 2, 16)
    # disjoint fake regions: qkv | cos | sin | q | k | v
    a = dict(qkv=A, cos=A + 3 * row * T, sin=A + 3 * row * T + T * D * 4, q=A + 3 * row * T + 2 * T * D * 4,
             T=T, H=H, D=D, dtype=vitattn.BF16)
    a["k"] = a["q"] + row * T
    a["v"] = a["k"] + row * T
    a.update(kw)
    return vitattn.check_args_qkv_rope(a["qkv"], a["cos"], a["sin"], a["q"], a["k"], a["v"], a["T"], a["H"], a["D"],
                                       a["dtype"])


def test_rope_valid_arguments_pass():
    assert check_rope() == 0
    assert check_rope(D=128, dtype=vitattn.F16) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(qkv=0), -1), (dict(sin=0), -1), (dict(v=0), -1),
    (dict(T=0), -2), (dict(H=0), -2), (dict(D=60), -3), (dict(D=8), -3), (dict(D=136), -3), (dict(dtype=5), -4),
    (dict(cos=A + 3 * 256 * 64 + 4), -5),
    (dict(q=A + 16), -6),                       # inside qkv
    (dict(k=A + 3 * 256 * 64 + 16), -6),        # inside the cos table
])
def test_rope_argument_errors(kw, code):
    assert check_rope(**kw) == code


def check_norm_rope(**kw):
    T, H, D = kw.get("T", 64), kw.get("H", 2), kw.get("D", 64)
    row = H * D * 2
    # disjoint fake regions: qkv | cos | sin | q | k | v | q_norm_w | k_norm_w
    a = dict(qkv=A, cos=A + 3 * row * T, sin=A + 3 * row * T + T * D * 4, q=A + 3 * row * T + 2 * T * D * 4,
             eps=1e-6, T=T, H=H, D=D, dtype=vitattn.BF16)
    a["k"] = a["q"] + row * T
    a["v"] = a["k"] + row * T
    a["qw"] = a["v"] + row * T
    a["kw"] = a["qw"] + D * 4
    a.update(kw)
    return vitattn.check_args_qkv_norm_rope(a["qkv"], a["cos"], a["sin"], a["qw"], a["kw"], a["eps"], a["q"], a["k"],
                                            a["v"], a["T"], a["H"], a["D"], a["dtype"])


def test_norm_rope_valid_arguments_pass():
    assert check_norm_rope() == 0
    assert check_norm_rope(D=128, dtype=vitattn.F16, eps=0.0) == 0
    assert check_norm_rope(kw=A) == 0                  # weights are read-only inputs: sharing qkv's memory is fine


V_END = A + 3 * 256 * 64 + 2 * 64 * 64 * 4 + 3 * 256 * 64   # one past v in the default layout


@pytest.mark.parametrize("kw,code", [
    (dict(qw=0), -1), (dict(kw=0), -1), (dict(qkv=0), -1),
    (dict(T=0), -2), (dict(D=60), -3), (dict(dtype=3), -4),
    (dict(qw=V_END + 4), -5), (dict(kw=V_END + 8), -5),
    (dict(eps=-1e-6), -9), (dict(eps=float("nan")), -9), (dict(eps=float("inf")), -9),
    (dict(qw=V_END - 64), -6),                         # overlaps the tail of v
    (dict(kw=A + 3 * 256 * 64 + 2 * 64 * 64 * 4 + 32), -6),   # inside q
    (dict(q=A + 16), -6),                              # the rope checks still apply
])
def test_norm_rope_argument_errors(kw, code):
    assert check_norm_rope(**kw) == code


# ---------------------------------------------------------------- grouped-query attention

def check_gqa(**kw):
    a = dict(q=Q, k=K, v=V, out=O, B=1, N=64, H=2, Hkv=1, D=64, scale=0.125, dtype=vitattn.BF16)
    a.update(kw)
    return vitattn.check_args_gqa(a["q"], a["k"], a["v"], a["out"], a["B"], a["N"], a["H"], a["Hkv"], a["D"],
                                  a["scale"], a["dtype"])


def test_gqa_valid_arguments_pass():
    assert check_gqa() == 0
    assert check_gqa(Hkv=2) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(k=0), -1), (dict(q=0), -1), (dict(Hkv=0), -2), (dict(H=3, Hkv=2), -2), (dict(Hkv=4), -2),
    (dict(D=70), -3), (dict(dtype=7), -4), (dict(v=V + 4), -5), (dict(out=K + 16), -6), (dict(out=Q), -6),
])
def test_gqa_argument_errors(kw, code):
    assert check_gqa(**kw) == code


# ---------------------------------------------------------------- cross lengths, causal mask, LSE

def check_ext(**kw):
    Lq, Lk, H, D = kw.get("Lq", 64), kw.get("Lk", 32), 2, 64
    qb, kb = Lq * H * D * 2, Lk * H * D * 2
    a = dict(q=A, out=A + qb, k=A + 2 * qb, v=A + 2 * qb + kb, lse=A + 2 * qb + 2 * kb, B=1, Lq=Lq, Lk=Lk, H=H, D=D,
             scale=0.125, dtype=vitattn.BF16)
    a.update(kw)
    return vitattn.check_args_ext(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["Lq"], a["Lk"], a["H"],
                                  a["D"], a["scale"], a["dtype"])


def test_ext_valid_arguments_pass():
    assert check_ext() == 0
    assert check_ext(lse=0) == 0
    assert check_ext(Lq=1, Lk=4096) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), -1), (dict(k=0), -1), (dict(Lk=0), -2), (dict(Lq=0), -2), (dict(D=60), -3),
    (dict(dtype=9), -4), (dict(lse=A + 2 * 64 * 256 + 2 * 32 * 256 + 4), -5), (dict(v=A + 8), -5),
    (dict(out=A + 2 * 64 * 256 + 16), -6), (dict(lse=A + 64 * 256 + 64), -6), (dict(scale=float("inf")), -9),
])
def test_ext_argument_errors(kw, code):
    assert check_ext(**kw) == code


def test_every_compute_entry_cites_the_passage_that_defines_it():
    """Each entry that launches work documents its operation with a reference
    to the page (by source path) that defines it."""
    text = open(HEADER).read()
    compute = {"vitattn_forward", "vitattn_forward_ext", "vitattn_forward_gqa", "vitattn_forward_varlen",
               "vitattn_qkv_rope", "vitattn_qkv_norm_rope", "vitattn_forward_host", "vitattn_forward_strided",
               "vitattn_qk_rope", "vitattn_qk_norm_rope"}
    seen = set()
    for m in re.finditer(r"/\*(.*?)\*/\s*VITATTN_API[^;(]*?\b(vitattn_\w+)\s*\(", text, re.S):
        comment, name = m.group(1), m.group(2)
        if name in compute:
            assert re.search(r"src/[\w/]+\.rs", comment), f"{name}: no source citation"
            seen.add(name)
    assert seen == compute


# ------------------------------------------------------------------ token-strided inputs

def check_strided(**kw):
    B, N, H, D = kw.get("B", 2), kw.get("N", 100), 2, 64
    row = H * D
    ts = kw.get("ts", 3 * row)
    span = ((B * N - 1) * ts + row) * 2  # bytes one strided input reaches
    qkv = A
    a = dict(q=qkv, k=qkv + 2 * row, v=qkv + 4 * row, out=A + span + 4 * row + 64, B=B, N=N, H=H, D=D,
             tq=ts, tk=ts, tv=ts, scale=0.125, dtype=vitattn.BF16)
    a.update(kw)
    return vitattn.check_args_strided(a["q"], a["k"], a["v"], a["out"], a["B"], a["N"], a["H"], a["D"], a["tq"],
                                      a["tk"], a["tv"], a["scale"], a["dtype"])


def test_strided_views_of_one_projection_pass():
    # q, k, v as the three column ranges of one packed [B, N, 3, H, D] projection
    assert check_strided() == 0
    # dense strides are the plain layout
    assert check_strided(ts=128, tq=128, tk=128, tv=128, k=A + 2 * 100 * 256 * 2, v=A + 4 * 100 * 256 * 2,
                         out=A + 6 * 100 * 256 * 2) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), -1), (dict(v=0), -1), (dict(tq=64), -2), (dict(tk=132), -2), (dict(tv=0), -2), (dict(B=0), -2),
    (dict(D=60), -3), (dict(dtype=5), -4), (dict(k=A + 2 * 128 + 8), -5), (dict(out=A + 96), -6),
    (dict(out=A + ((2 * 100 - 1) * 384 + 128) * 2 + 2 * 128 - 16), -6), (dict(scale=float("nan")), -9),
])
def test_strided_argument_errors(kw, code):
    assert check_strided(**kw) == code


def test_qk_rope_checks_need_no_v_and_refuse_aliasing():
    T, H, D = 16, 2, 64
    qkv = A
    inb = T * 3 * H * D * 2
    cs, sn = A + inb, A + inb + T * D * 4
    q, k = sn + T * D * 4, sn + T * D * 4 + T * H * D * 2
    assert vitattn.check_args_qk_rope(qkv, cs, sn, q, k, T, H, D, vitattn.BF16) == 0
    assert vitattn.check_args_qk_rope(qkv, cs, sn, q, q, T, H, D, vitattn.BF16) == -6   # q and k overlap
    assert vitattn.check_args_qk_rope(qkv, cs, sn, qkv + 64, k, T, H, D, vitattn.BF16) == -6  # q inside qkv
    assert vitattn.check_args_qk_rope(qkv, cs, sn, 0, k, T, H, D, vitattn.BF16) == -1
    assert vitattn.check_args_qk_rope(qkv, cs, sn, q, k, T, H, 72, 7) == -4


@pytest.mark.parametrize("B,H,D", [(1, 16, 64), (2, 16, 128), (3, 12, 80), (1, 1, 64), (1, 3, 16), (7, 5, 32),
                                   (16, 4, 64), (32, 16, 64), (9, 4, 64), (1, 40, 128), (4, 2, 128)])
def test_host_plan_covers_every_image_and_head_once(B, H, D):
    """The host-buffer entry's cut of a batch: every (image, head) in exactly
    one group, at most 8 groups of images or 16 of heads, and when heads are
    cut each copied row of a group is at least 512 bytes wide."""
    per_chunk, G, n = vitattn.host_plan(B, H, D)
    assert 1 <= n <= (16 if G > 1 else 8)
    seen = np.zeros((B, H), dtype=int)
    for c in range(n):
        if G > 1:
            b0, nb, h0 = c // G, 1, (c % G) * H // G
            nh = (c % G + 1) * H // G - h0
            assert nh * D * 2 >= 512
        else:
            b0, nb, h0, nh = c * per_chunk, min(per_chunk, B - c * per_chunk), 0, H
        assert nb >= 1 and nh >= 1
        seen[b0:b0 + nb, h0:h0 + nh] += 1
    assert np.all(seen == 1)
    if B >= 8:
        assert G == 1  # whole images when there are enough of them
