"""GPU parity for the packed-projection path: the q/k-only prologue
(``vitattn_qk_rope``, ``vitattn_qk_norm_rope``) and the attention reading q, k
and v through token strides (``vitattn_forward_strided``), so that v is read
straight out of the packed ``[B, N, 3, H, D]`` projection instead of being
copied (inferencelayer ``src/vision_gpu.rs``, ``VIS_QKV_ROPE`` doc: the
projection output is q | k | v per token).

The strided attention computes exactly what ``vitattn_forward`` computes on
the same values, so it must match the dense entry bit for bit; the q/k-only
prologues must match the full prologues' q and k bit for bit; and the chain
must meet the attention tolerance (max |O - O_ref| <= 1e-2, relative
Frobenius <= 4e-3) against the fp64 oracle chain.
"""
import numpy as np
import pytest

import oracle
from vit_bidirectional_attention_b200 import synth, vitattn

pytestmark = pytest.mark.gpu


def tdt(dtype):
    import torch

    return torch.bfloat16 if dtype == synth.BF16 else torch.float16


def to_dev(bits, dtype):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy()).view(tdt(dtype)).cuda()


def bits_of(t):
    import torch

    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def as_f64(t, dtype):
    return synth.bits_to_float32(bits_of(t), dtype).astype(np.float64)


@pytest.mark.parametrize("B,N,H,D,dtype", [
    (1, 64, 2, 64, synth.BF16), (2, 200, 3, 80, synth.BF16), (1, 196, 16, 72, synth.F16),
    (3, 333, 2, 128, synth.BF16), (2, 1000, 4, 64, synth.F16),
])
def test_strided_views_match_the_dense_entry_bit_for_bit(cuda_device, B, N, H, D, dtype):
    import torch

    qkv = synth.make_qkv_packed(B * N, H, D, dtype, seed=9000 + N + D, std=1.3)
    t = to_dev(qkv, dtype).view(B, N, 3, H, D)
    q, k, v = t.unbind(2)                      # token stride 3*H*D, read in place
    got = vitattn.forward_strided(q, k, v, checked=True)
    dense = vitattn.forward(q.contiguous(), k.contiguous(), v.contiguous(), checked=True)
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(got), bits_of(dense))
    ref = oracle.attention(*(qkv[:, j].reshape(B, N, H, D) for j in range(3)), 1.0 / np.sqrt(D), dtype)
    g = as_f64(got, dtype)
    assert np.max(np.abs(g - ref)) <= 1e-2
    assert np.linalg.norm(g - ref) / np.linalg.norm(ref) <= 4e-3


def test_mixed_strides(cuda_device):
    # q dense, k with a padded token stride, v from a packed projection
    import torch

    B, N, H, D = 2, 300, 2, 64
    qkv = synth.make_qkv_packed(B * N, H, D, synth.BF16, seed=9101)
    t = to_dev(qkv, synth.BF16).view(B, N, 3, H, D)
    q = t[:, :, 0].contiguous()
    kpad = torch.zeros((B, N, H * D + 24), dtype=torch.bfloat16, device="cuda")
    kpad[:, :, : H * D] = t[:, :, 1].reshape(B, N, H * D)
    k = torch.as_strided(kpad, (B, N, H, D), (N * (H * D + 24), H * D + 24, D, 1))
    v = t[:, :, 2]
    got = vitattn.forward_strided(q, k, v, scale=0.2, checked=True)
    dense = vitattn.forward(q, k.contiguous(), v.contiguous(), scale=0.2, checked=True)
    assert np.array_equal(bits_of(got), bits_of(dense))


@pytest.mark.parametrize("H,D", [(4, 64), (19, 64), (7, 32), (5, 80)])
@pytest.mark.parametrize("normed", [False, True])
def test_qk_prologue_matches_the_full_prologue(cuda_device, normed, H, D):
    import torch

    T = 777
    qkv = synth.make_qkv_packed(T, H, D, synth.BF16, seed=9200, std=1.5)
    cs, sn = synth.rope_tables_2d(28, 28, D)
    cs, sn = cs[:T].copy(), sn[:T].copy()
    tq = to_dev(qkv, synth.BF16)
    tc, ts = torch.from_numpy(cs).cuda(), torch.from_numpy(sn).cuda()
    if normed:
        qw = torch.from_numpy(synth.make_norm_weights(D, 9201)[0]).cuda()
        kw = torch.from_numpy(synth.make_norm_weights(D, 9201)[1]).cuda()
        q, k, v = vitattn.qk_rope(tq, tc, ts, qw, kw, 1e-6)
        fq, fk, _ = vitattn.qkv_norm_rope(tq, tc, ts, qw, kw, 1e-6)
    else:
        q, k, v = vitattn.qk_rope(tq, tc, ts)
        fq, fk, _ = vitattn.qkv_rope(tq, tc, ts)
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(q), bits_of(fq))
    assert np.array_equal(bits_of(k), bits_of(fk))
    assert v.data_ptr() == tq.data_ptr() + 2 * H * D * 2   # v is the projection itself
    assert np.array_equal(bits_of(v), qkv[:, 2])


@pytest.mark.parametrize("name", ["layer_batched", "layer_packed_batched"])
def test_layer_workload_sampled_parity_at_full_size(cuda_device, name):
    """The layer bench workloads at full size (32 images of 32 x 32 patches, 16
    heads, D = 64, bf16, the bench's seeded projection and tables) through the
    calls the bench times: the full prologue and the dense attention, or the
    q/k-only prologue and the attention reading v from the projection; 1024
    seeded token-head rows against the oracle chain."""
    import torch

    w = synth.LAYER[name]
    pw = synth.PrologueWorkload(w.name, w.images, w.grid, w.H, w.D, w.dtype, index=w.index)
    qkv, cs, sn = synth.make_prologue(pw)
    B, N, H, D = w.images, w.N, w.H, w.D
    tq = to_dev(qkv, w.dtype)
    tc, ts = torch.from_numpy(cs).cuda(), torch.from_numpy(sn).cuda()
    if w.packed:
        q, k, v = vitattn.qk_rope(tq, tc, ts)
        out = vitattn.forward_strided(q.view(B, N, H, D), k.view(B, N, H, D), v.view(B, N, H, D), scale=w.scale,
                                      checked=True)
    else:
        q, k, v = vitattn.qkv_rope(tq, tc, ts)
        out = vitattn.forward(q.view(B, N, H, D), k.view(B, N, H, D), v.view(B, N, H, D), scale=w.scale, checked=True)
    torch.cuda.synchronize()
    rq, rk, _ = oracle.qkv_rope(qkv, cs, sn, w.dtype)
    oq, ok = (synth.round_to_bits(x.astype(np.float32), w.dtype) for x in (rq, rk))
    rows = np.sort(np.random.Generator(np.random.PCG64(9310)).choice(B * N * H, 1024, replace=False))
    got = as_f64(out, w.dtype).reshape(B * N * H, D)[rows]
    ref = oracle.attention_rows(oq.reshape(B, N, H, D), ok.reshape(B, N, H, D),
                                np.ascontiguousarray(qkv[:, 2]).reshape(B, N, H, D), w.scale, w.dtype, rows)
    assert np.max(np.abs(got - ref)) <= 1e-2
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 4e-3


def test_packed_layer_chain_against_the_oracle(cuda_device):
    """qk_rope, then the attention reading v from the projection: the layer of
    the batched workload at 4 images, against the oracle chain."""
    import torch

    B, N, H, D = 4, 1024, 16, 64
    qkv = synth.make_qkv_packed(B * N, H, D, synth.BF16, seed=9300)
    cs, sn = synth.rope_tables_2d(32, 32, D)
    cs, sn = np.tile(cs, (B, 1)), np.tile(sn, (B, 1))
    tq = to_dev(qkv, synth.BF16)
    q, k, v = vitattn.qk_rope(tq, torch.from_numpy(cs).cuda(), torch.from_numpy(sn).cuda())
    out = vitattn.forward_strided(q.view(B, N, H, D), k.view(B, N, H, D), v.view(B, N, H, D), checked=True)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.qkv_rope(qkv, cs, sn, synth.BF16)
    oq, ok = (synth.round_to_bits(x.astype(np.float32), synth.BF16) for x in (rq, rk))
    # flat token-head rows (b*N + i)*H + h, a seeded sample
    rows = np.sort(np.random.Generator(np.random.PCG64(9301)).choice(B * N * H, 1024, replace=False))
    got = as_f64(out, synth.BF16).reshape(B * N * H, D)[rows]
    ref = oracle.attention_rows(oq.reshape(B, N, H, D), ok.reshape(B, N, H, D),
                                np.ascontiguousarray(qkv[:, 2]).reshape(B, N, H, D), 0.125, synth.BF16, rows)
    assert np.max(np.abs(got - ref)) <= 1e-2
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 4e-3
