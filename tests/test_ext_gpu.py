"""GPU parity for cross-length attention with the aligned causal mask and the
LSE output (``vitattn_forward_ext``; hanzo-ml ``src/vulkan_backend.rs``,
``flash_attn_gpu``: query i sees keys j <= i + (Lk - Lq) when ``causal``),
against the fp64 oracle's ``attention_ext``.

Tolerances: the output as for the dense path (max-abs 1e-2, relative
Frobenius 4e-3); the LSE within 1e-3 absolute (it is the log of the f32 sum
of probabilities from the exp2 unit, each within a few f32 ulps of the exact
value, and the rescale factors); rows that see no key exactly 0 with LSE
-inf.
"""
import math

import numpy as np
import pytest

import oracle
from vit_bidirectional_attention_b200 import synth, vitattn

pytestmark = pytest.mark.gpu

FORCE_TWO_TILES, FORCE_ONE_TILE, TINY_GRID = 2, 4, 8


def to_dev(bits, dtype):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy())
    return t.view(torch.bfloat16 if dtype == synth.BF16 else torch.float16).cuda()


def from_dev(t, dtype):
    import torch

    return synth.bits_to_float32(t.view(torch.int16).cpu().numpy().view(np.uint16), dtype).astype(np.float64)


def inputs(B, Lq, Lk, H, D, dtype, seed, std=1.0):
    rng = np.random.Generator(np.random.PCG64(seed))
    q = synth.round_to_bits(rng.standard_normal((B, Lq, H, D), dtype=np.float32) * np.float32(std), dtype)
    k = synth.round_to_bits(rng.standard_normal((B, Lk, H, D), dtype=np.float32) * np.float32(std), dtype)
    v = synth.round_to_bits(rng.standard_normal((B, Lk, H, D), dtype=np.float32), dtype)
    return q, k, v


def run_ext(q, k, v, scale, causal, dtype, flags=0):
    import torch

    tq, tk, tv = (to_dev(x, dtype) for x in (q, k, v))
    B, Lq, H, D = q.shape
    out = torch.full_like(tq, float("nan"))
    lse = torch.full((B, H, Lq), float("nan"), dtype=torch.float32, device="cuda")
    rc = vitattn.forward_ext_ptr(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Lq,
                                 k.shape[1], H, D, scale, causal, dtype, torch.cuda.current_stream().cuda_stream,
                                 checked=True, flags=flags)
    assert rc == 0, vitattn.strerror(rc)
    return from_dev(out, dtype), lse.cpu().numpy().astype(np.float64)


def check(got, ref, lse, lse_ref, what):
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    max_abs = float(np.max(np.abs(got - ref)))
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    assert max_abs <= 1e-2 and rel <= 4e-3, f"{what}: max_abs={max_abs:.3e} rel_frob={rel:.3e}"
    none = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), none), f"{what}: rows without keys"
    if (~none).any():
        err = float(np.max(np.abs(lse[~none] - lse_ref[~none])))
        assert err <= 1e-3, f"{what}: lse err {err:.3e}"


SHAPES = [(300, 300), (200, 500), (500, 200), (1, 129), (129, 1), (257, 256), (640, 640)]


@pytest.mark.parametrize("flags", [FORCE_TWO_TILES, FORCE_ONE_TILE])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Lq,Lk", SHAPES)
@pytest.mark.parametrize("D,dtype", [(64, synth.BF16), (128, synth.F16), (80, synth.BF16)])
def test_ext_parity(cuda_device, Lq, Lk, causal, D, dtype, flags):
    q, k, v = inputs(2, Lq, Lk, 2, D, dtype, seed=9500 + Lq * 3 + Lk + D + int(causal), std=1.3)
    scale = 1.0 / math.sqrt(D)
    got, lse = run_ext(q, k, v, scale, causal, dtype, flags)
    ref, lse_ref = oracle.attention_ext(q, k, v, scale, dtype, causal=causal)
    check(got, ref, lse, lse_ref, f"Lq={Lq} Lk={Lk} causal={causal} D={D} flags={flags}")


def test_causal_1024_with_peaky_logits(cuda_device):
    q, k, v = inputs(1, 1024, 1024, 4, 64, synth.BF16, seed=9600, std=2.5)
    got, lse = run_ext(q, k, v, 0.125, True, synth.BF16)
    ref, lse_ref = oracle.attention_ext(q, k, v, 0.125, synth.BF16, causal=True)
    check(got, ref, lse, lse_ref, "causal 1024")


def test_unmasked_same_length_is_the_plain_entry_bitwise(cuda_device):
    import torch

    q, k, v = synth.random_qkv(2, 300, 3, 64, synth.BF16, seed=9700)
    got, _ = run_ext(q, k, v, 0.125, False, synth.BF16)
    tq, tk, tv = (to_dev(x, synth.BF16) for x in (q, k, v))
    plain = vitattn.forward(tq, tk, tv, scale=0.125, checked=True)
    assert np.array_equal(got, from_dev(plain, synth.BF16))


def test_python_entry_returns_out_and_lse(cuda_device):
    q, k, v = inputs(1, 100, 250, 4, 72, synth.F16, seed=9800)
    tq, tk, tv = (to_dev(x, synth.F16) for x in (q, k, v))
    out, lse = vitattn.forward_ext(tq, tk, tv, causal=True, with_lse=True, checked=True)
    ref, lse_ref = oracle.attention_ext(q, k, v, 1.0 / math.sqrt(72), synth.F16, causal=True)
    check(from_dev(out, synth.F16), ref, lse.cpu().numpy().astype(np.float64), lse_ref, "python entry")


@pytest.mark.parametrize("flags", [FORCE_TWO_TILES | TINY_GRID, FORCE_ONE_TILE | TINY_GRID])
@pytest.mark.parametrize("Lq,Lk", [(512, 512), (256, 640), (384, 384)])
def test_causal_many_heads_and_groups(cuda_device, Lq, Lk, flags):
    """Causal launches with several heads and query groups per head (work
    items of different key-block counts, each head's longest group first).
    The tiny-grid flag must not change anything for them."""
    q, k, v = inputs(3, Lq, Lk, 3, 64, synth.BF16, seed=9900 + Lq + Lk + flags)
    got, lse = run_ext(q, k, v, 0.125, True, synth.BF16, flags)
    ref, lse_ref = oracle.attention_ext(q, k, v, 0.125, synth.BF16, causal=True)
    check(got, ref, lse, lse_ref, f"Lq={Lq} Lk={Lk} flags={flags}")


def test_causal_launch_with_more_items_than_sms(cuda_device):
    """4 x 1024 x 16 x 64: 256 work items of 2 to 8 key blocks, more than the
    SMs (one CTA per item)."""
    q, k, v = inputs(4, 1024, 1024, 16, 64, synth.BF16, seed=9950)
    got, lse = run_ext(q, k, v, 0.125, True, synth.BF16)
    ref, lse_ref = oracle.attention_ext(q, k, v, 0.125, synth.BF16, causal=True)
    check(got, ref, lse, lse_ref, "causal 4x1024x16x64")


@pytest.mark.parametrize("B,H,N,D", [(2, 16, 1024, 64), (3, 7, 777, 64), (1, 40, 2048, 64), (2, 9, 1280, 128),
                                     (2, 5, 896, 80)])
def test_causal_whole_slices_against_the_oracle(cuda_device, B, H, N, D):
    """Causal launches with many items of 1 to 16 key blocks: every row of two
    (b, h) slices against the oracle (output and LSE), and the same bits with
    the tiny-grid flag, which causal launches ignore (one CTA per item).  777
    tokens leave a lone last query tile."""
    q, k, v = inputs(B, N, N, H, D, synth.BF16, seed=9970 + N + H + D)
    scale = D ** -0.5
    tiny, lse_l = run_ext(q, k, v, scale, True, synth.BF16, TINY_GRID | FORCE_TWO_TILES)
    got = tiny.reshape(B, N, H, D)
    # every query row of two (b, h) slices: whole causal rows of the oracle
    for b, h in ((0, 0), (B - 1, H - 1)):
        o, lse_o = oracle.attention_ext(q[b:b + 1, :, h:h + 1], k[b:b + 1, :, h:h + 1], v[b:b + 1, :, h:h + 1],
                                        scale, synth.BF16, causal=True)
        check(got[b:b + 1, :, h:h + 1], o, lse_l[b:b + 1, h:h + 1], lse_o, f"causal {B}x{N}x{H}x{D} ({b},{h})")
    wide, lse_w = run_ext(q, k, v, scale, True, synth.BF16, FORCE_TWO_TILES)
    assert np.array_equal(tiny, wide) and np.array_equal(lse_l, lse_w)


def test_batched_causal_workload_sampled_parity_at_full_size(cuda_device):
    """The causal bench workload at full size (32 x 1024 x 16 x 64 bf16, causal,
    LSE) in the launch the bench times (default flags: one CTA per item):
    every row of six (b, h) slices, the first, the last and four seeded ones,
    against the oracle, output and LSE."""
    w = synth.WORKLOADS["batched_causal"]
    q, k, v = synth.make_qkv(w)
    got, lse = run_ext(q, k, v, w.scale, True, w.dtype)
    rng = np.random.Generator(np.random.PCG64(9990))
    picks = [(0, 0), (w.B - 1, w.H - 1)] + [(int(rng.integers(w.B)), int(rng.integers(w.H))) for _ in range(4)]
    for b, h in picks:
        o, lse_o = oracle.attention_ext(q[b:b + 1, :, h:h + 1], k[b:b + 1, :, h:h + 1], v[b:b + 1, :, h:h + 1],
                                        w.scale, w.dtype, causal=True)
        check(got[b:b + 1, :, h:h + 1], o, lse[b:b + 1, h:h + 1], lse_o, f"batched_causal ({b},{h})")
