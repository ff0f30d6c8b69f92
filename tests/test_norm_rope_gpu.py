"""GPU parity for the prologue with a per-head q/k RMS norm
(``vitattn_qkv_norm_rope``; inferencelayer ``src/vision_gpu.rs``,
``GLM_QKV_QKNORM_ROPE``: split the packed qkv, normalise each head's q and k
row with a per-element weight, then rotate), against the fp64 oracle
``qkv_norm_rope``.

Error bound.  The kernel computes x' = inv * (x*A + p*B) in f32, with
A = w*cos, B = sign*w_p*sin formed once per token and inv the inverse root:
- the head's sum of squares takes at most 9 roundings along any path (4 per
  lane, then a butterfly of up to 5 levels), and all its terms are positive:
  relative error <= 9u, with u = 2^-24;
- the mean plus eps is one fma with 1/D (2u), and rsqrtf adds at most 2 ulp
  (4u), so inv is within about 10u;
- A, B and p*B take one rounding each, then the fma and the product with inv
  take one more each.
Every q/k element must therefore lie within one unit in the last place (of
the storage dtype) of the exact value, plus 2^-19 * (|y*c| + |y_p*s|), where
y is the normed row.  The 2^-19 allows 32u, about twice the ~15u the steps
above add up to.  At least 99% of the elements must be the exact
round-to-nearest result, and v must be a bit-exact copy.
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
    mant = 7 if dtype == synth.BF16 else 10
    emin = -126 if dtype == synth.BF16 else -14
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** emin)))
    return 2.0 ** (e - mant)


def weights(D, seed):
    return synth.make_norm_weights(D, seed)


def tables(T, D):
    w = max(1, int(np.sqrt(T)))
    cs, sn = synth.rope_tables_2d((T + w - 1) // w, w, D)
    return cs[:T].copy(), sn[:T].copy()


def run(qkv, cs, sn, qw, kw, eps, dtype):
    import torch

    dev = [torch.from_numpy(x).cuda() for x in (cs, sn, qw, kw)]
    q, k, v = vitattn.qkv_norm_rope(to_dev(qkv, dtype), *dev, eps)
    torch.cuda.synchronize()
    return q, k, v


def check(qkv, cs, sn, qw, kw, eps, dtype, got, rows=None):
    """Element-wise bound and round-to-nearest share against the oracle;
    ``rows`` restricts the check to a token sample."""
    sel = slice(None) if rows is None else rows
    x, c, s = qkv[sel], cs[sel], sn[sel]
    rq, rk, _ = oracle.qkv_norm_rope(x, c, s, qw, kw, eps, dtype)
    one, zero = np.ones_like(c), np.zeros_like(c)
    yq, yk, _ = oracle.qkv_norm_rope(x, one, zero, qw, kw, eps, dtype)    # the normed rows, unrotated
    D = x.shape[-1]
    for t, ref, y, name in ((got[0], rq, yq, "q"), (got[1], rk, yk, "k")):
        g = synth.bits_to_float32(bits_of(t)[sel], dtype).astype(np.float64)
        yp = np.concatenate([-y[..., D // 2:], y[..., :D // 2]], axis=-1)
        lim = ulp(ref, dtype) + 2.0 ** -19 * (np.abs(y * c[:, None, :]) + np.abs(yp * s[:, None, :]))
        err = np.abs(g - ref)
        assert np.all(err <= lim * 1.0000001), f"{name}: worst {np.max(err / lim):.3f} of the bound"
        exact = synth.round_to_bits(ref.astype(np.float32), dtype)
        assert np.mean(bits_of(t)[sel] == exact) > 0.99, f"{name}: too few round-to-nearest results"
    assert np.array_equal(bits_of(got[2])[sel], qkv[sel][:, 2])


@pytest.mark.parametrize("T,H,D,dtype,std,eps", [
    (1, 1, 16, synth.BF16, 1.0, 1e-6), (5, 3, 64, synth.BF16, 1.7, 1e-6), (1000, 2, 72, synth.F16, 1.0, 1e-5),
    (333, 16, 80, synth.BF16, 0.3, 1e-6), (257, 4, 128, synth.F16, 2.0, 0.0), (196, 16, 72, synth.F16, 1.0, 1e-6),
    (64, 5, 24, synth.BF16, 40.0, 1e-6), (77, 7, 64, synth.BF16, 0.05, 0.5),
    (50, 9, 32, synth.F16, 1.0, 1e-6), (40, 11, 48, synth.BF16, 1.3, 1e-6), (31, 17, 64, synth.BF16, 1.0, 1e-6),
    (9, 3, 16, synth.F16, 1.0, 1e-6), (23, 5, 40, synth.BF16, 1.0, 1e-6), (19, 6, 56, synth.F16, 0.7, 1e-6),
])
def test_norm_prologue_within_bound(cuda_device, T, H, D, dtype, std, eps):
    qkv = synth.make_qkv_packed(T, H, D, dtype, seed=8500 + T + D, std=std)
    cs, sn = tables(T, D)
    qw, kw = weights(D, 8600 + D)
    got = run(qkv, cs, sn, qw, kw, eps, dtype)
    check(qkv, cs, sn, qw, kw, eps, dtype, got)


def test_norm_prologue_zero_rows_with_eps_are_zero(cuda_device):
    T, H, D = 9, 3, 64
    qkv = synth.make_qkv_packed(T, H, D, synth.BF16, seed=8700)
    qkv[2, 0, 1] = 0          # one q head row of zeros
    qkv[5, 1, :] = 0          # every k head of one token
    cs, sn = tables(T, D)
    qw, kw = weights(D, 8701)
    got = run(qkv, cs, sn, qw, kw, 1e-6, synth.BF16)
    q, k = bits_of(got[0]), bits_of(got[1])
    assert not (q[2, 1] & 0x7FFF).any() and not (k[5] & 0x7FFF).any()
    check(qkv, cs, sn, qw, kw, 1e-6, synth.BF16, got)


def test_norm_prologue_differs_from_the_plain_prologue(cuda_device):
    """The same inputs through both prologues: unit weights, eps = 0 and unit-RMS
    rows would make them agree, so ordinary inputs must not."""
    import torch

    T, H, D = 50, 4, 64
    qkv = synth.make_qkv_packed(T, H, D, synth.BF16, seed=8800, std=3.0)
    cs, sn = tables(T, D)
    qw, kw = weights(D, 8801)
    got = run(qkv, cs, sn, qw, kw, 1e-6, synth.BF16)
    plain = vitattn.qkv_rope(to_dev(qkv, synth.BF16), torch.from_numpy(cs).cuda(), torch.from_numpy(sn).cuda())
    torch.cuda.synchronize()
    assert not np.array_equal(bits_of(got[0]), bits_of(plain[0]))
    assert np.array_equal(bits_of(got[2]), bits_of(plain[2]))


def test_norm_prologue_on_the_batched_shape(cuda_device):
    """The rope_norm_batched workload (32 x 1024 tokens, 16 heads, D = 64, bf16)
    as the bench runs it: a seeded sample of 2048 tokens checked element by
    element, the first and last among them; v checked in full."""
    w = synth.PROLOGUE["rope_norm_batched"]
    qkv, cs, sn = synth.make_prologue(w)
    qw, kw = synth.make_norm_weights(w.D, w.seed + 1000)
    got = run(qkv, cs, sn, qw, kw, w.eps, w.dtype)
    idx = np.sort(np.random.Generator(np.random.PCG64(8901)).choice(w.T, 2048, replace=False))
    idx[0], idx[-1] = 0, w.T - 1
    check(qkv, cs, sn, qw, kw, w.eps, w.dtype, got, rows=idx)
    assert np.array_equal(bits_of(got[2]), qkv[:, 2])


def test_norm_prologue_then_dense_attention(cuda_device):
    B, N, H, D = 2, 196, 4, 64
    qkv = synth.make_qkv_packed(B * N, H, D, synth.BF16, seed=9000, std=1.2)
    cs, sn = synth.rope_tables_2d(14, 14, D)
    cs, sn = np.tile(cs, (B, 1)), np.tile(sn, (B, 1))
    qw, kw = weights(D, 9001)
    q, k, v = run(qkv, cs, sn, qw, kw, 1e-6, synth.BF16)
    out = vitattn.forward(q.view(B, N, H, D), k.view(B, N, H, D), v.view(B, N, H, D), scale=0.125, checked=True)
    got = synth.bits_to_float32(bits_of(out), synth.BF16).astype(np.float64)
    rq, rk, rv = oracle.qkv_norm_rope(qkv, cs, sn, qw, kw, 1e-6, synth.BF16)
    oq, ok, ov = (synth.round_to_bits(x.astype(np.float32), synth.BF16).reshape(B, N, H, D) for x in (rq, rk, rv))
    ref = oracle.attention(oq, ok, ov, 0.125, synth.BF16)
    assert np.max(np.abs(got - ref)) <= 1e-2
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 4e-3


def test_norm_prologue_rejects_bad_eps_before_launch(cuda_device):
    import torch

    qkv = to_dev(synth.make_qkv_packed(4, 2, 64, synth.BF16, seed=9100), synth.BF16)
    cs, sn = (torch.from_numpy(x).cuda() for x in tables(4, 64))
    qw, kw = (torch.from_numpy(x).cuda() for x in weights(64, 9101))
    for eps in (-1.0, float("nan")):
        with pytest.raises(vitattn.VitAttnError):
            vitattn.qkv_norm_rope(qkv, cs, sn, qw, kw, eps)
