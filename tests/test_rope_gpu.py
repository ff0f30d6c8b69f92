"""GPU parity for the attention's prologue (``vitattn_qkv_rope``): split a
packed QKV projection and rotate q and k with per-token cos/sin tables
(inferencelayer ``src/vision_gpu.rs``, ``VIS_QKV_ROPE``), against the fp64
oracle ``qkv_rope``.

The kernel computes x*c + r*s in f32 (r*s rounded, then one fma) and rounds
once to the storage dtype.  So every q/k element must lie within one unit in
the last place (of that dtype) of the exact fp64 value plus the f32
evaluation error, 2^-23 * (|x*c| + |r*s|) (it matters only where the two
products nearly cancel); at least 99% of the elements must be the exact
round-to-nearest result; and v is a bit-exact copy.  Chained with the attention
kernel, the result must meet the attention tolerance against the oracle
chain.
"""
import numpy as np
import pytest

import oracle
from vit_bidirectional_attention_b200 import synth, vitattn

pytestmark = pytest.mark.gpu


def to_dev(bits, dtype):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy())
    return t.view(torch.bfloat16 if dtype == synth.BF16 else torch.float16).cuda()


def bits_of(t):
    import torch

    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def ulp(x, dtype):
    """One unit in the last place of the storage dtype at magnitude |x|."""
    mant = 7 if dtype == synth.BF16 else 10
    emin = -126 if dtype == synth.BF16 else -14
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** emin)))
    return 2.0 ** (e - mant)


def bound(qkv_x, cs, sn, dtype, ref):
    """Allowed |gpu - ref| per element: one dtype ulp plus the f32 evaluation error."""
    x = oracle.widen(np.ascontiguousarray(qkv_x), dtype)
    D = x.shape[-1]
    r = np.concatenate([-x[..., D // 2:], x[..., :D // 2]], axis=-1)
    mag = np.abs(x * cs[:, None, :]) + np.abs(r * sn[:, None, :])
    return ulp(ref, dtype) + 2.0 ** -23 * mag


def run_rope(qkv, cs, sn, dtype):
    import torch

    T, _, H, D = qkv.shape
    tq = to_dev(qkv, dtype)
    tc, ts = torch.from_numpy(cs).cuda(), torch.from_numpy(sn).cuda()
    q, k, v = vitattn.qkv_rope(tq, tc, ts)
    torch.cuda.synchronize()
    return q, k, v


def grid_tables(T, D, w=None):
    w = w or max(1, int(np.sqrt(T)))
    cs, sn = synth.rope_tables_2d((T + w - 1) // w, w, D)
    return cs[:T].copy(), sn[:T].copy()


@pytest.mark.parametrize("T,H,D,dtype", [
    (1, 1, 16, synth.BF16), (5, 3, 64, synth.BF16), (1000, 2, 72, synth.F16),
    (333, 16, 80, synth.BF16), (257, 4, 128, synth.F16), (196, 16, 72, synth.F16), (64, 5, 24, synth.BF16),
    (50, 9, 32, synth.F16), (40, 11, 48, synth.BF16), (31, 17, 64, synth.BF16), (9, 3, 16, synth.F16),
    (23, 5, 40, synth.BF16), (19, 6, 56, synth.F16),
])
def test_prologue_within_one_ulp(cuda_device, T, H, D, dtype):
    qkv = synth.make_qkv_packed(T, H, D, dtype, seed=8000 + T + D, std=1.7)
    cs, sn = grid_tables(T, D)
    q, k, v = run_rope(qkv, cs, sn, dtype)
    rq, rk, rv = oracle.qkv_rope(qkv, cs, sn, dtype)
    for j, (got, ref, name) in enumerate(((q, rq, "q"), (k, rk, "k"))):
        g = synth.bits_to_float32(bits_of(got), dtype).astype(np.float64)
        err = np.abs(g - ref)
        lim = bound(qkv[:, j], cs, sn, dtype, ref)
        assert np.all(err <= lim * 1.0000001), f"{name}: worst {np.max(err / lim):.3f} of the bound"
        exact = synth.round_to_bits(ref.astype(np.float32), dtype)
        assert np.mean(bits_of(got) == exact) > 0.99, f"{name}: too few round-to-nearest results"
    assert np.array_equal(bits_of(v), qkv[:, 2])


def test_prologue_on_the_batched_shape(cuda_device):
    """32 x 1024 tokens, 16 heads, D = 64 (the batched workload's QKV): a seeded
    sample of 2048 tokens checked element by element."""
    T, H, D = 32 * 1024, 16, 64
    qkv = synth.make_qkv_packed(T, H, D, synth.BF16, seed=8100)
    cs, sn = synth.rope_tables_2d(32, 32, D)
    cs, sn = np.tile(cs, (32, 1)), np.tile(sn, (32, 1))
    q, k, v = run_rope(qkv, cs, sn, synth.BF16)
    idx = np.sort(np.random.Generator(np.random.PCG64(8101)).choice(T, 2048, replace=False))
    idx[0], idx[-1] = 0, T - 1
    rq, rk, _ = oracle.qkv_rope(qkv[idx], cs[idx], sn[idx], synth.BF16)
    for j, (got, ref) in enumerate(((q, rq), (k, rk))):
        g = synth.bits_to_float32(bits_of(got)[idx], synth.BF16).astype(np.float64)
        lim = bound(qkv[idx, j], cs[idx], sn[idx], synth.BF16, ref)
        assert np.all(np.abs(g - ref) <= lim * 1.0000001)
        exact = synth.round_to_bits(ref.astype(np.float32), synth.BF16)
        assert np.mean(bits_of(got)[idx] == exact) > 0.99
    assert np.array_equal(bits_of(v), qkv[:, 2])


def _oracle_chain_inputs(qkv, cs, sn, dtype):
    rq, rk, rv = oracle.qkv_rope(qkv, cs, sn, dtype)
    return (synth.round_to_bits(x.astype(np.float32), dtype) for x in (rq, rk, rv))


def test_prologue_then_dense_attention(cuda_device):
    import torch

    B, N, H, D = 2, 196, 4, 64
    qkv = synth.make_qkv_packed(B * N, H, D, synth.BF16, seed=8200, std=1.2)
    cs, sn = synth.rope_tables_2d(14, 14, D)
    cs, sn = np.tile(cs, (B, 1)), np.tile(sn, (B, 1))
    q, k, v = run_rope(qkv, cs, sn, synth.BF16)
    out = vitattn.forward(q.view(B, N, H, D), k.view(B, N, H, D), v.view(B, N, H, D), scale=0.125, checked=True)
    got = synth.bits_to_float32(bits_of(out), synth.BF16).astype(np.float64)
    oq, ok, ov = _oracle_chain_inputs(qkv, cs, sn, synth.BF16)
    ref = oracle.attention(oq.reshape(B, N, H, D), ok.reshape(B, N, H, D), ov.reshape(B, N, H, D), 0.125,
                           synth.BF16)
    assert np.max(np.abs(got - ref)) <= 1e-2
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 4e-3


def test_prologue_then_ragged_attention(cuda_device):
    lens = [196, 400]
    T, H, D = sum(lens), 2, 80
    qkv = synth.make_qkv_packed(T, H, D, synth.F16, seed=8300)
    c1, s1 = synth.rope_tables_2d(14, 14, D)
    c2, s2 = synth.rope_tables_2d(20, 20, D)
    cs, sn = np.concatenate([c1, c2]), np.concatenate([s1, s2])
    q, k, v = run_rope(qkv, cs, sn, synth.F16)
    cu = [0, 196, 596]
    out = vitattn.forward_varlen(q, k, v, cu, checked=True)
    got = synth.bits_to_float32(bits_of(out), synth.F16).astype(np.float64)
    oq, ok, ov = _oracle_chain_inputs(qkv, cs, sn, synth.F16)
    ref = oracle.attention_varlen(oq, ok, ov, cu, 1.0 / np.sqrt(D), synth.F16)
    assert np.max(np.abs(got - ref)) <= 1e-2
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 4e-3
