"""Pins for the fp64 oracle: checks against things other than the oracle itself.

The oracle computes, per (batch, head), O = softmax(scale * Q K^T) V with no
mask (hf2q ``src/inference/vision/vit_gpu.rs``: doc of ``vit_attention_gpu``
and ``vit_attention_scores_gpu``; inferencelayer ``src/vision_gpu.rs``:
``vis_attn_coop_src`` doc).  Each test below pins it to a closed form, an
invariant of the definition, a hand-derived fixture, exhaustive conversion
tables, or an independent library routine, so that a dropped term, a wrong
sign, a transposed operand or a mixed-up index fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from vit_bidirectional_attention_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_form_cases.txt")


def rnd(shape, seed, std=1.0):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(size=shape) * std


# ---------------------------------------------------------------- conversions

def test_widen_f16_exhaustive_matches_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.widen(bits, oracle.F16)
    want = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])


def test_widen_bf16_exhaustive_matches_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.widen(bits, oracle.BF16)
    want = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])


@pytest.mark.parametrize("dtype", [synth.BF16, synth.F16])
def test_generator_rounding_is_round_to_nearest_even(dtype):
    x = rnd(200_000, 5, std=3.0).astype(np.float32)
    x[:4] = [0.0, -0.0, 1e-8, 65504.0]
    bits = synth.round_to_bits(x, dtype)
    tdt = torch.bfloat16 if dtype == synth.BF16 else torch.float16
    want = torch.from_numpy(x).to(tdt).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, want)


# ---------------------------------------------------------------- fixtures

def _parse_golden():
    cases, cur = [], None
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        tok = line.split()
        if tok[0] == "case":
            kv = dict(t.split("=") for t in tok[2:])
            cur = {"name": tok[1], "N": int(kv["N"]), "D": int(kv["D"]), "scale": float(kv["scale"])}
        elif tok[0] in ("q", "k", "v"):
            cur[tok[0]] = np.array([float(t) for t in tok[1:]])
        elif tok[0] == "o":
            env = {"sig": lambda x: 1.0 / (1.0 + math.exp(-x)), "exp": math.exp}
            cur["o"] = np.array([eval(t, {"__builtins__": {}}, env) for t in tok[1:]])
        elif tok[0] == "end":
            cases.append(cur)
    return cases


GOLDEN_CASES = _parse_golden()


@pytest.mark.parametrize("case", GOLDEN_CASES, ids=[c["name"] for c in GOLDEN_CASES])
@pytest.mark.parametrize("dtype", [oracle.F64, oracle.BF16, oracle.F16])
def test_hand_derived_closed_forms(case, dtype):
    N, D = case["N"], case["D"]
    shape = (1, N, 1, D)
    q, k, v = (case[n].reshape(shape) for n in "qkv")
    if dtype != oracle.F64:
        q, k, v = (synth.round_to_bits(x.astype(np.float32), dtype) for x in (q, k, v))
    out = oracle.attention(q, k, v, case["scale"], dtype)
    np.testing.assert_allclose(out.reshape(-1), case["o"], rtol=0, atol=1e-15)


def test_golden_file_has_cases():
    assert len(GOLDEN_CASES) >= 3


# ---------------------------------------------------------------- closed forms

@pytest.mark.parametrize("scale", [0.125, 1.0, -3.0, 40.0])
def test_single_token_returns_v(scale):
    q, k, v = (rnd((2, 1, 3, 16), s) for s in (1, 2, 3))
    out = oracle.attention(q, k, v, scale, oracle.F64)
    assert np.array_equal(out, v)


def test_zero_scale_gives_mean_of_v():
    q, k, v = (rnd((2, 37, 3, 24), s) for s in (4, 5, 6))
    out = oracle.attention(q, k, v, 0.0, oracle.F64)
    want = np.broadcast_to(v.mean(axis=1, keepdims=True), v.shape)
    np.testing.assert_allclose(out, want, rtol=0, atol=1e-14)


def test_identical_keys_give_mean_of_v():
    B, N, H, D = 1, 50, 2, 32
    q, v = rnd((B, N, H, D), 7), rnd((B, N, H, D), 8)
    k = np.broadcast_to(rnd((B, 1, H, D), 9), (B, N, H, D)).copy()
    out = oracle.attention(q, k, v, 0.3, oracle.F64)
    want = np.broadcast_to(v.mean(axis=1, keepdims=True), v.shape)
    np.testing.assert_allclose(out, want, rtol=0, atol=1e-14)


def test_all_ones_v_gives_ones():
    q, k = rnd((2, 70, 2, 16), 10, std=2.0), rnd((2, 70, 2, 16), 11, std=2.0)
    v = np.ones_like(q)
    out = oracle.attention(q, k, v, 0.25, oracle.F64)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-14)


def test_two_keys_logistic_form():
    # N = 2: O_i = sig(s_i0 - s_i1) v_0 + sig(s_i1 - s_i0) v_1 with s = scale * q.k
    q, k, v = (rnd((1, 2, 1, 8), s) for s in (12, 13, 14))
    scale = 0.7
    out = oracle.attention(q, k, v, scale, oracle.F64)[0, :, 0]
    sig = lambda x: 1.0 / (1.0 + math.exp(-x))
    for i in range(2):
        d = scale * (float(q[0, i, 0] @ k[0, 0, 0]) - float(q[0, i, 0] @ k[0, 1, 0]))
        want = sig(d) * v[0, 0, 0] + sig(-d) * v[0, 1, 0]
        np.testing.assert_allclose(out[i], want, rtol=0, atol=1e-15)


def test_dominant_key_selects_its_value():
    B, N, H, D = 1, 40, 1, 16
    q = np.zeros((B, N, H, D)); q[..., 0] = 1.0
    k = rnd((B, N, H, D), 15) * 0.01
    k[0, 17, 0, 0] = 100.0
    v = rnd((B, N, H, D), 16)
    out = oracle.attention(q, k, v, 1.0, oracle.F64)
    np.testing.assert_allclose(out[0, :, 0], np.broadcast_to(v[0, 17, 0], (N, D)), rtol=0, atol=1e-30)


def test_huge_logits_stay_finite():
    # the max shift keeps exp in range; without it exp(2000) overflows
    q, k, v = (rnd((1, 30, 1, 8), s) for s in (17, 18, 19))
    out = oracle.attention(q, k, v, 500.0, oracle.F64)
    assert np.all(np.isfinite(out))
    P = oracle.probs(q, k, 500.0, oracle.F64, 0, 0)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-14)


def test_all_scores_far_below_zero_stay_finite():
    # every score near -1000: exp(s) underflows unless the row maximum is subtracted
    g = np.random.Generator(np.random.PCG64(48))
    q = np.abs(g.standard_normal((1, 25, 2, 8))) + 1.0
    k = np.abs(g.standard_normal((1, 25, 2, 8))) + 1.0
    v = g.standard_normal((1, 25, 2, 8))
    out = oracle.attention(q, k, v, -80.0, oracle.F64)
    assert np.all(np.isfinite(out))
    # the least negative score dominates: compare against the row argmax of q.k scaled
    P = oracle.probs(q, k, -80.0, oracle.F64, 0, 1)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    s = -80.0 * np.einsum("id,jd->ij", q[0, :, 1], k[0, :, 1])
    assert np.array_equal(P.argmax(axis=1), s.argmax(axis=1))


# ---------------------------------------------------------------- invariants

def test_probability_rows_sum_to_one_and_produce_out():
    q, k, v = (rnd((2, 45, 3, 24), s) for s in (20, 21, 22))
    out = oracle.attention(q, k, v, 0.4, oracle.F64)
    for b in range(2):
        for h in range(3):
            P = oracle.probs(q, k, 0.4, oracle.F64, b, h)
            assert np.all(P >= 0)
            np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-14)
            np.testing.assert_allclose(P @ v[b, :, h], out[b, :, h], rtol=0, atol=1e-13)


def test_joint_key_value_permutation_invariance():
    q, k, v = (rnd((2, 33, 2, 16), s) for s in (23, 24, 25))
    perm = np.random.Generator(np.random.PCG64(26)).permutation(33)
    a = oracle.attention(q, k, v, 0.5, oracle.F64)
    b = oracle.attention(q, k[:, perm], v[:, perm], 0.5, oracle.F64)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)


def test_query_permutation_permutes_output():
    q, k, v = (rnd((1, 29, 2, 16), s) for s in (27, 28, 29))
    perm = np.random.Generator(np.random.PCG64(30)).permutation(29)
    a = oracle.attention(q, k, v, 0.5, oracle.F64)
    b = oracle.attention(q[:, perm], k, v, 0.5, oracle.F64)
    np.testing.assert_allclose(a[:, perm], b, rtol=0, atol=1e-15)


def test_affine_in_v():
    q, k, v = (rnd((1, 31, 2, 8), s) for s in (31, 32, 33))
    c = rnd((8,), 34)
    a = oracle.attention(q, k, v, 0.6, oracle.F64)
    b = oracle.attention(q, k, 2.5 * v + c, 0.6, oracle.F64)
    np.testing.assert_allclose(b, 2.5 * a + c, rtol=0, atol=1e-13)


def test_common_key_shift_leaves_output_unchanged():
    # K[j] -> K[j] + c shifts every score of row i by scale*q_i.c: softmax ignores it.
    # Small integers keep every input exact in bf16.
    g = np.random.Generator(np.random.PCG64(35))
    q = g.integers(-2, 3, size=(1, 20, 2, 16)).astype(np.float32)
    k = g.integers(-2, 3, size=(1, 20, 2, 16)).astype(np.float32)
    v = g.integers(-4, 5, size=(1, 20, 2, 16)).astype(np.float32)
    c = g.integers(-3, 4, size=(16,)).astype(np.float32)
    bits = lambda x: synth.round_to_bits(x, synth.BF16)
    a = oracle.attention(bits(q), bits(k), bits(v), 0.25, oracle.BF16)
    b = oracle.attention(bits(q), bits(k + c), bits(v), 0.25, oracle.BF16)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)


def test_heads_and_batches_are_independent_slices():
    B, N, H, D = 2, 19, 3, 8
    q, k, v = (rnd((B, N, H, D), s) for s in (36, 37, 38))
    full = oracle.attention(q, k, v, 0.9, oracle.F64)
    for b in range(B):
        for h in range(H):
            sl = lambda x: np.ascontiguousarray(x[b:b + 1, :, h:h + 1, :])
            one = oracle.attention(sl(q), sl(k), sl(v), 0.9, oracle.F64)
            assert np.array_equal(one[0, :, 0], full[b, :, h])


# ---------------------------------------------------------------- library routine

@pytest.mark.parametrize("shape,scale", [((2, 65, 3, 64), 0.125), ((1, 130, 2, 72), 1 / math.sqrt(72)),
                                         ((3, 17, 1, 80), -0.2), ((1, 5, 4, 16), 2.0)])
def test_matches_torch_sdpa_float64(shape, scale):
    q, k, v = (rnd(shape, 40 + s, std=1.5) for s in range(3))
    out = oracle.attention(q, k, v, scale, oracle.F64)
    t = lambda x: torch.from_numpy(x).permute(0, 2, 1, 3)  # [B,H,N,D]
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), scale=scale)
    ref = ref.permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-13)


# ---------------------------------------------------------------- internal consistency

@pytest.mark.parametrize("dtype", [oracle.BF16, oracle.F16])
def test_formulations_agree_on_tiny(dtype):
    w = synth.WORKLOADS["tiny"]
    q, k, v = synth.random_qkv(1, 48, 2, 16, dtype, seed=44)
    a = oracle.attention(q, k, v, 0.25, dtype, mode=oracle.MODE_TWO_PASS)
    b = oracle.attention(q, k, v, 0.25, dtype, mode=oracle.MODE_LSE)
    c = oracle.attention(q, k, v, 0.25, dtype, mode=oracle.MODE_BRUTE)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
    np.testing.assert_allclose(a, c, rtol=0, atol=1e-12)
    assert w.N == 64


def test_bits_path_equals_widened_f64_path():
    q, k, v = synth.random_qkv(2, 40, 3, 24, synth.F16, seed=45)
    a = oracle.attention(q, k, v, 0.3, oracle.F16)
    b = oracle.attention(*(oracle.widen(x, oracle.F16) for x in (q, k, v)), 0.3, oracle.F64)
    assert np.array_equal(a, b)


def test_rows_entry_matches_full_output():
    q, k, v = synth.random_qkv(2, 70, 3, 16, synth.BF16, seed=46)
    full = oracle.attention(q, k, v, 0.25, oracle.BF16)
    rows = synth.sample_rows((2, 70, 3), 50, seed=47)
    part = oracle.attention_rows(q, k, v, 0.25, oracle.BF16, rows)
    assert np.array_equal(part, full.reshape(-1, 16)[rows])


def test_bad_arguments_raise():
    q = np.zeros((1, 4, 1, 8), dtype=np.uint16)
    with pytest.raises(RuntimeError):
        oracle.attention_rows(q, q, q, 1.0, oracle.BF16, np.array([4], dtype=np.int64))
    with pytest.raises(TypeError):
        oracle.attention(q.astype(np.float32), q, q, 1.0, oracle.BF16)


def test_workload_table_matches_stated_shapes():
    w = synth.WORKLOADS
    assert (w["small_vit"].N, w["small_vit"].H, w["small_vit"].D) == (196, 16, 72)
    assert (w["doc_page"].N, w["doc_page"].D) == (912, 80)
    assert (w["batched"].B, w["batched"].N, w["batched"].D) == (32, 1024, 64)
    assert (w["high_res"].B, w["high_res"].N, w["high_res"].D) == (2, 16384, 128)
    assert w["batched"].flops == 4 * 32 * 16 * 1024 ** 2 * 64


def test_rank8_recipe_reaches_logit_std_4():
    # measured on a reduced-N copy of the high-res recipe (same D, same alpha)
    w = synth.Workload("hr_small", 1, 2048, 2, 128, synth.BF16, rank8_logit_std=4.0, index=4)
    q, k, _ = synth.make_qkv(w)
    qf, kf = (synth.bits_to_float32(x, synth.BF16).astype(np.float64) for x in (q, k))
    s = np.einsum("nd,md->nm", qf[0, :, 0], kf[0, :, 0]) / math.sqrt(128)
    assert 3.6 < s.std() < 4.4


# ---------------------------------------------------------------- ragged (multi-image) batches

def _block_diag_brute(qf, kf, vf, cu, scale):
    """Independent formulation: one softmax over the whole packed token axis
    with every key outside the query's own segment masked to -inf."""
    T, H, D = qf.shape
    seg = np.zeros(T, np.int64)
    for s, (a, b) in enumerate(zip(cu, cu[1:])):
        seg[a:b] = s
    out = np.zeros((T, H, D))
    for h in range(H):
        logits = scale * (qf[:, h, :] @ kf[:, h, :].T)
        logits[seg[:, None] != seg[None, :]] = -np.inf
        logits -= logits.max(axis=1, keepdims=True)
        w = np.exp(logits)
        w /= w.sum(axis=1, keepdims=True)
        out[:, h, :] = w @ vf[:, h, :]
    return out


@pytest.mark.parametrize("cu", [[0, 5], [0, 1, 4, 9], [0, 3, 3, 7, 8], [0, 0, 6, 6, 13]])
def test_varlen_oracle_matches_block_diagonal_masked_softmax(cu):
    T, H, D = cu[-1], 2, 8
    q, k, v = (synth.round_to_bits(rnd((T, H, D), 90 + i, 1.5).astype(np.float32), synth.BF16) for i in range(3))
    got = oracle.attention_varlen(q, k, v, cu, 0.4, oracle.BF16)
    qf, kf, vf = (oracle.widen(x, oracle.BF16) for x in (q, k, v))
    np.testing.assert_allclose(got, _block_diag_brute(qf, kf, vf, cu, 0.4), rtol=0, atol=1e-12)


def test_varlen_oracle_equal_segments_is_the_dense_batch():
    B, N, H, D = 3, 7, 2, 16
    q, k, v = synth.random_qkv(B, N, H, D, synth.F16, seed=91)
    dense = oracle.attention(q, k, v, 0.25, oracle.F16)
    packed = oracle.attention_varlen(q.reshape(B * N, H, D), k.reshape(B * N, H, D), v.reshape(B * N, H, D),
                                     [0, N, 2 * N, 3 * N], 0.25, oracle.F16)
    assert np.array_equal(packed.reshape(B, N, H, D), dense)


def test_varlen_oracle_segments_do_not_see_each_other():
    cu = [0, 4, 10]
    q, k, v = (synth.round_to_bits(rnd((10, 2, 8), 92 + i).astype(np.float32), synth.BF16) for i in range(3))
    a = oracle.attention_varlen(q, k, v, cu, 0.5, oracle.BF16)
    k2, v2 = k.copy(), v.copy()
    k2[4:] = synth.round_to_bits(rnd((6, 2, 8), 95).astype(np.float32), synth.BF16)
    v2[4:] = synth.round_to_bits(rnd((6, 2, 8), 96).astype(np.float32), synth.BF16)
    b = oracle.attention_varlen(q, k2, v2, cu, 0.5, oracle.BF16)
    assert np.array_equal(a[:4], b[:4])
    assert not np.array_equal(a[4:], b[4:])


def test_varlen_oracle_rejects_bad_offsets():
    q = np.zeros((4, 1, 8), np.uint16)
    for cu in ([1, 4], [0, 3, 2, 4], [0, 3]):
        with pytest.raises(ValueError):
            oracle.attention_varlen(q, q, q, cu, 1.0, oracle.BF16)


def test_varlen_rows_match_the_full_varlen_output():
    cu = [0, 3, 3, 11, 16]
    q, k, v = (synth.round_to_bits(rnd((16, 3, 8), 97 + i).astype(np.float32), synth.F16) for i in range(3))
    full = oracle.attention_varlen(q, k, v, cu, 0.3, oracle.F16).reshape(16 * 3, 8)
    rows = np.array([47, 0, 9, 10, 30, 8, 33])
    assert np.array_equal(oracle.attention_varlen_rows(q, k, v, cu, 0.3, oracle.F16, rows), full[rows])


# ---------------------------------------------------------------- QKV split + rotary embedding prologue

def _rope_case(T, H, D, seed, dtype=synth.BF16):
    qkv = synth.round_to_bits(rnd((T, 3, H, D), seed).astype(np.float32), dtype)
    theta = rnd((T, D // 2), seed + 1)
    ang = np.concatenate([theta, theta], axis=1)       # the two halves of a pair share an angle
    return qkv, np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def test_rope_is_a_complex_rotation_of_each_pair():
    """Independent form: pair (x_d, x_{d+D/2}) as x_d + i x_{d+D/2}, multiplied
    by e^{i theta_d}."""
    qkv, c, s = _rope_case(7, 3, 16, 120)
    q, k, v = oracle.qkv_rope(qkv, c, s, oracle.BF16)
    x = oracle.widen(qkv, oracle.BF16)
    for src, got in ((x[:, 0], q), (x[:, 1], k)):
        z = src[..., :8] + 1j * src[..., 8:]
        e = c[:, None, :8].astype(np.float64) + 1j * s[:, None, :8].astype(np.float64)
        zr = z * e
        np.testing.assert_allclose(got[..., :8], zr.real, rtol=0, atol=1e-12)
        np.testing.assert_allclose(got[..., 8:], zr.imag, rtol=0, atol=1e-12)
    assert np.array_equal(v, x[:, 2])


def test_rope_identity_and_quarter_turn():
    qkv, _, _ = _rope_case(4, 2, 8, 121, synth.F16)
    ones, zeros = np.ones((4, 8), np.float32), np.zeros((4, 8), np.float32)
    x = oracle.widen(qkv, oracle.F16)
    q, k, _ = oracle.qkv_rope(qkv, ones, zeros, oracle.F16)
    assert np.array_equal(q, x[:, 0]) and np.array_equal(k, x[:, 1])
    q, k, _ = oracle.qkv_rope(qkv, zeros, ones, oracle.F16)      # rotate_half itself
    assert np.array_equal(q[..., :4], -x[:, 0, :, 4:]) and np.array_equal(q[..., 4:], x[:, 0, :, :4])


def test_rope_preserves_pair_norms_and_dot_products_shift():
    qkv, c, s = _rope_case(9, 2, 32, 122)
    q, k, _ = oracle.qkv_rope(qkv, c, s, oracle.BF16)
    x = oracle.widen(qkv, oracle.BF16)
    n0 = x[:, 0, :, :16] ** 2 + x[:, 0, :, 16:] ** 2
    n1 = q[..., :16] ** 2 + q[..., 16:] ** 2
    np.testing.assert_allclose(n1, n0, rtol=1e-6)   # cos/sin are float32: |c + i s| = 1 to ~1e-7


def test_rope_hand_fixture():
    # D = 4, one head, one token: q = (1, 2, 3, 4), angle pi/2 on pair 0 and 0 on pair 1
    qkv = np.zeros((1, 3, 1, 4), np.float64)
    qkv[0, 0, 0] = [1, 2, 3, 4]
    qkv[0, 1, 0] = [5, 6, 7, 8]
    qkv[0, 2, 0] = [9, 10, 11, 12]
    c = np.array([[0.0, 1.0, 0.0, 1.0]])
    s = np.array([[1.0, 0.0, 1.0, 0.0]])
    q, k, v = oracle.qkv_rope(qkv, c, s, oracle.F64)
    assert q[0, 0].tolist() == [-3.0, 2.0, 1.0, 4.0]
    assert k[0, 0].tolist() == [-7.0, 6.0, 5.0, 8.0]
    assert v[0, 0].tolist() == [9.0, 10.0, 11.0, 12.0]


# ---------------------------------------------------------------- prologue with q/k RMS norm

def test_norm_rope_unit_weights_give_unit_rms_per_head():
    """w = 1, eps = 0, identity tables: every output q and k head row has mean
    square exactly 1 (the mean is over D, not a sum), v is untouched."""
    qkv, _, _ = _rope_case(5, 3, 24, 130)
    ones, zeros = np.ones((5, 24), np.float32), np.zeros((5, 24), np.float32)
    w = np.ones(24)
    q, k, v = oracle.qkv_norm_rope(qkv, ones, zeros, w, w, 0.0, oracle.BF16)
    for t in (q, k):
        np.testing.assert_allclose(np.mean(t * t, axis=-1), 1.0, rtol=0, atol=1e-13)
    assert np.array_equal(v, oracle.widen(qkv, oracle.BF16)[:, 2])


def test_norm_rope_is_scale_invariant_without_eps():
    qkv, c, s = _rope_case(4, 2, 16, 131)
    x = oracle.widen(qkv, oracle.BF16)
    w = rnd((16,), 132)
    a = oracle.qkv_norm_rope(x, c, s, w, w[::-1], 0.0, oracle.F64)
    b = oracle.qkv_norm_rope(x * 37.5, c, s, w, w[::-1], 0.0, oracle.F64)
    for i in (0, 1):
        np.testing.assert_allclose(b[i], a[i], rtol=1e-13, atol=1e-13)


def test_norm_rope_constant_row_with_eps_closed_form():
    """x = 3 everywhere, eps = 7: mean square 9, 3 / sqrt(9 + 7) = 3/4, so
    under identity tables q = 0.75 * wq and k = 0.75 * wk (eps inside the
    root and added to the mean; the two weight vectors kept apart)."""
    D = 8
    qkv = np.full((1, 3, 2, D), 3.0)
    wq = np.arange(1.0, D + 1.0)
    wk = -np.arange(D, 0.0, -1.0)
    q, k, v = oracle.qkv_norm_rope(qkv, np.ones((1, D)), np.zeros((1, D)), wq, wk, 7.0, oracle.F64)
    assert np.array_equal(q, np.broadcast_to(0.75 * wq, q.shape))
    assert np.array_equal(k, np.broadcast_to(0.75 * wk, k.shape))
    assert np.array_equal(v, qkv[:, 2])


@pytest.mark.parametrize("j", [0, 2, 5, 7])
def test_norm_rope_one_hot_under_quarter_turn_pins_the_order(j):
    """x = -2 e_j, cos = 0, sin = 1 (the rotation is rotate_half itself),
    eps = 0: the norm gives -sqrt(D) e_j * w_j, then rotate_half moves it to
    j + D/2 (same sign) or j - D/2 (negated).  Rotating first and normalising
    after would pick up w at the destination instead of w_j."""
    D, half = 8, 4
    qkv = np.zeros((1, 3, 1, D))
    qkv[0, 0, 0, j] = -2.0
    qkv[0, 1, 0, j] = 5.0
    wq = np.array([1.5, -2.0, 0.25, 3.0, 0.5, 4.0, -1.0, 2.5])
    wk = wq[::-1].copy()
    q, k, _ = oracle.qkv_norm_rope(qkv, np.zeros((1, D)), np.ones((1, D)), wq, wk, 0.0, oracle.F64)
    dest, sign = (j + half, 1.0) if j < half else (j - half, -1.0)
    want_q = np.zeros(D)
    want_q[dest] = sign * -math.sqrt(D) * wq[j]
    want_k = np.zeros(D)
    want_k[dest] = sign * math.sqrt(D) * wk[j]
    np.testing.assert_allclose(q[0, 0], want_q, rtol=0, atol=1e-14)
    np.testing.assert_allclose(k[0, 0], want_k, rtol=0, atol=1e-14)


def test_norm_rope_with_unit_weights_commutes_with_a_pair_rotation():
    """With w = 1 the norm is a scalar per head and the rope (pairs sharing an
    angle) preserves the head's norm, so normalising after the rotation gives
    the same result; per element, the output is the rotated input over its RMS."""
    qkv, c, s = _rope_case(6, 2, 32, 133)
    x = oracle.widen(qkv, oracle.BF16)
    w = np.ones(32)
    q, k, _ = oracle.qkv_norm_rope(qkv, c, s, w, w, 0.0, oracle.BF16)
    zq = x[:, 0, :, :16] + 1j * x[:, 0, :, 16:]
    e = c[:, None, :16].astype(np.float64) + 1j * s[:, None, :16].astype(np.float64)
    rms = np.sqrt(np.mean(x[:, 0] ** 2, axis=-1))[..., None]
    zr = zq * e / rms
    np.testing.assert_allclose(q[..., :16], zr.real, rtol=0, atol=1e-6)  # |c + i s| = 1 to float32 rounding
    np.testing.assert_allclose(q[..., 16:], zr.imag, rtol=0, atol=1e-6)
    assert np.all(np.isfinite(k))


def test_norm_rope_hand_fixture():
    """D = 4 by hand.  q = (1, 2, 3, 4): mean square 30/4 = 7.5, so with
    weights (2, 1, 1, 3) the normed row is (2, 2, 3, 12)/sqrt(7.5); the quarter
    turn on pair 0 (angle pi/2) and none on pair 1 then give
    (-3, 2, 2, 12)/sqrt(7.5).  k = (5, 6, 7, 8) with unit weights and eps = 0:
    mean square 174/4 = 43.5, output (-7, 6, 5, 8)/sqrt(43.5)."""
    qkv = np.zeros((1, 3, 1, 4))
    qkv[0, 0, 0] = [1, 2, 3, 4]
    qkv[0, 1, 0] = [5, 6, 7, 8]
    qkv[0, 2, 0] = [9, 10, 11, 12]
    c = np.array([[0.0, 1.0, 0.0, 1.0]])
    s = np.array([[1.0, 0.0, 1.0, 0.0]])
    q, k, v = oracle.qkv_norm_rope(qkv, c, s, np.array([2.0, 1.0, 1.0, 3.0]), np.ones(4), 0.0, oracle.F64)
    np.testing.assert_allclose(q[0, 0], np.array([-3.0, 2.0, 2.0, 12.0]) / math.sqrt(7.5), rtol=1e-15, atol=0)
    np.testing.assert_allclose(k[0, 0], np.array([-7.0, 6.0, 5.0, 8.0]) / math.sqrt(43.5), rtol=1e-15, atol=0)
    assert v[0, 0].tolist() == [9.0, 10.0, 11.0, 12.0]


def test_norm_rope_zero_row_with_eps_is_zero():
    qkv = np.zeros((2, 3, 1, 16))
    q, k, _ = oracle.qkv_norm_rope(qkv, np.ones((2, 16)), np.zeros((2, 16)), np.ones(16), np.ones(16), 1e-6,
                                   oracle.F64)
    assert not q.any() and not k.any()


# ---------------------------------------------------------------- grouped-query attention

@pytest.mark.parametrize("H,Hkv", [(4, 2), (6, 3), (4, 1), (3, 3)])
def test_gqa_oracle_matches_per_head_brute_force(H, Hkv):
    """Independent form: per (b, h) softmax over keys of kv head h // (H/Hkv)."""
    B, N, D = 2, 5, 8
    q = synth.round_to_bits(rnd((B, N, H, D), 130).astype(np.float32), synth.BF16)
    k = synth.round_to_bits(rnd((B, N, Hkv, D), 131).astype(np.float32), synth.BF16)
    v = synth.round_to_bits(rnd((B, N, Hkv, D), 132).astype(np.float32), synth.BF16)
    got = oracle.attention_gqa(q, k, v, 0.35, oracle.BF16)
    qf, kf, vf = (oracle.widen(x, oracle.BF16) for x in (q, k, v))
    g = H // Hkv
    for b in range(B):
        for h in range(H):
            s = 0.35 * qf[b, :, h] @ kf[b, :, h // g].T
            w = np.exp(s - s.max(axis=1, keepdims=True))
            w /= w.sum(axis=1, keepdims=True)
            np.testing.assert_allclose(got[b, :, h], w @ vf[b, :, h // g], rtol=0, atol=1e-12)


def test_gqa_oracle_heads_of_a_group_share_keys_and_values():
    q1 = synth.round_to_bits(rnd((1, 6, 1, 8), 133).astype(np.float32), synth.F16)
    q = np.concatenate([q1, q1, q1, q1], axis=2)          # 4 identical query heads
    k = synth.round_to_bits(rnd((1, 6, 2, 8), 134).astype(np.float32), synth.F16)
    v = synth.round_to_bits(rnd((1, 6, 2, 8), 135).astype(np.float32), synth.F16)
    o = oracle.attention_gqa(q, k, v, 0.5, oracle.F16)
    assert np.array_equal(o[:, :, 0], o[:, :, 1]) and np.array_equal(o[:, :, 2], o[:, :, 3])
    assert not np.array_equal(o[:, :, 0], o[:, :, 2])


def test_gqa_oracle_rejects_bad_head_counts():
    q = np.zeros((1, 2, 6, 8), np.uint16)
    with pytest.raises(ValueError):
        oracle.attention_gqa(q, np.zeros((1, 2, 4, 8), np.uint16), np.zeros((1, 2, 4, 8), np.uint16), 1.0,
                             oracle.BF16)


# ---------------------------------------------------------------- cross lengths, aligned causal mask, LSE

def _ext_inputs(B, Lq, Lk, H, D, seed, dtype=synth.BF16):
    rng = np.random.Generator(np.random.PCG64(seed))
    q = synth.round_to_bits(rng.standard_normal((B, Lq, H, D), dtype=np.float32), dtype)
    k = synth.round_to_bits(rng.standard_normal((B, Lk, H, D), dtype=np.float32), dtype)
    v = synth.round_to_bits(rng.standard_normal((B, Lk, H, D), dtype=np.float32), dtype)
    return q, k, v


def test_ext_without_mask_equals_the_plain_oracle_and_its_probabilities():
    q, k, v = _ext_inputs(2, 9, 9, 3, 8, 140)
    out, lse = oracle.attention_ext(q, k, v, 0.4, oracle.BF16)
    np.testing.assert_allclose(out, oracle.attention(q, k, v, 0.4, oracle.BF16), rtol=0, atol=1e-12)
    qf, kf = oracle.widen(q, oracle.BF16), oracle.widen(k, oracle.BF16)
    for b in range(2):
        for h in range(3):
            s = 0.4 * qf[b, :, h] @ kf[b, :, h].T
            # p = exp(s - lse) is the softmax the plain oracle exposes
            np.testing.assert_allclose(np.exp(s - lse[b, h][:, None]), oracle.probs(q, k, 0.4, oracle.BF16, b, h),
                                       rtol=0, atol=1e-12)


def test_ext_causal_rows_see_the_aligned_prefix():
    Lq, Lk = 5, 8                                     # offset Lk - Lq = 3
    q, k, v = _ext_inputs(1, Lq, Lk, 2, 8, 141)
    out, lse = oracle.attention_ext(q, k, v, 0.3, oracle.BF16, causal=True)
    for i in range(Lq):
        n = i + 3 + 1                                 # keys 0 .. i + 3
        sub_out, sub_lse = oracle.attention_ext(q[:, i:i + 1], k[:, :n], v[:, :n], 0.3, oracle.BF16)
        np.testing.assert_allclose(out[:, i], sub_out[:, 0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[:, :, i], sub_lse[:, :, 0], rtol=0, atol=1e-12)


def test_ext_causal_first_row_is_v0_and_lse_is_its_score():
    q, k, v = _ext_inputs(1, 6, 6, 1, 8, 142)
    out, lse = oracle.attention_ext(q, k, v, 0.5, oracle.BF16, causal=True)
    vf, qf, kf = (oracle.widen(x, oracle.BF16) for x in (v, q, k))
    assert np.array_equal(out[0, 0, 0], vf[0, 0, 0])
    assert lse[0, 0, 0] == 0.5 * float(qf[0, 0, 0] @ kf[0, 0, 0])


def test_ext_rows_that_see_no_key_are_zero_with_lse_minus_inf():
    q, k, v = _ext_inputs(1, 7, 4, 2, 8, 143)           # offset -3: rows 0..2 see nothing
    out, lse = oracle.attention_ext(q, k, v, 0.5, oracle.BF16, causal=True)
    assert np.all(out[:, :3] == 0.0) and np.all(np.isneginf(lse[:, :, :3]))
    assert np.all(np.isfinite(lse[:, :, 3:]))


def test_ext_lse_is_the_log_of_the_exponential_sum():
    q, k, v = _ext_inputs(1, 4, 6, 1, 8, 144)
    _, lse = oracle.attention_ext(q, k, v, 0.25, oracle.BF16)
    qf, kf = oracle.widen(q, oracle.BF16), oracle.widen(k, oracle.BF16)
    direct = np.log(np.exp(0.25 * qf[0, :, 0] @ kf[0, :, 0].T).sum(axis=1))
    np.testing.assert_allclose(lse[0, 0], direct, rtol=0, atol=1e-12)
