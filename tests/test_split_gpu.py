"""Split items on the GPU: when a grid of one-tile items cannot fill the SMs
with two tiles each, a query tile's key blocks are split over the CTA's two
softmax warpgroups, each with its own running (m, l, O), and merged at the
end like one more online-softmax step (the running-output rescale of
inferencelayer ``src/vision_gpu.rs``, doc of ``vis_attn_coop_src``, "The
obstacle, and the way round it").

Every case is checked against the fp64 oracle at the usual tolerance
(max |O_gpu - O_ref| <= 1e-2, relative Frobenius <= 4e-3; LSE within 1e-3),
and against the same launch with splitting turned off (a test-only flag),
which differs only in summation order: within the same bound of each other.
Shapes cover even and odd key-block counts (an odd count leaves the upper
half one block past the keys, masked whole), ragged tails, every padded head
dim, both dtypes, cross lengths, grouped-query heads and the LSE output.
"""
import math

import numpy as np
import pytest

import oracle
from vit_bidirectional_attention_b200 import synth, vitattn

pytestmark = pytest.mark.gpu

NO_SPLIT = 16
SPLIT_FROM_TWO = 32  # split from two key blocks on (the default starts at four)
FORCE_ONE_TILE = 4


def to_dev(bits, dtype):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy())
    return t.view(torch.bfloat16 if dtype == synth.BF16 else torch.float16).cuda()


def from_dev(t, dtype):
    import torch

    bits = t.view(torch.int16).cpu().numpy().view(np.uint16)
    return synth.bits_to_float32(bits, dtype).astype(np.float64)


def close(got, ref, what, max_abs=1e-2, rel=4e-3):
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = float(np.max(np.abs(got - ref)))
    r = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    assert err <= max_abs and r <= rel, f"{what}: max_abs={err:.3e} rel_frob={r:.3e}"


def run_ext(q, k, v, scale, dtype, flags, want_lse=True):
    import torch

    tq, tk, tv = (to_dev(x, dtype) for x in (q, k, v))
    B, Lq, H, D = q.shape
    out = torch.full_like(tq, float("nan"))
    lse = torch.full((B, H, Lq), float("nan"), dtype=torch.float32, device="cuda")
    rc = vitattn.forward_ext_ptr(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), out.data_ptr(),
                                 lse.data_ptr() if want_lse else 0, B, Lq, k.shape[1], H, D, scale, False, dtype,
                                 torch.cuda.current_stream().cuda_stream, flags=flags)
    assert rc == 0, vitattn.strerror(rc)
    return from_dev(out, dtype), lse.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("N,D,dtype", [
    (129, 64, synth.BF16),   # 2 key blocks, a 1-key tail
    (300, 80, synth.BF16),   # 3 blocks: the upper half's second block lies past the keys
    (384, 128, synth.F16),   # 3 full blocks
    (912, 80, synth.BF16),   # the document page: 8 blocks
    (196, 72, synth.F16),    # the small ViT block: 2 blocks
    (640, 16, synth.BF16), (500, 32, synth.F16), (700, 48, synth.BF16), (1000, 96, synth.F16),
    (777, 112, synth.BF16),
])
def test_split_against_the_oracle_and_the_unsplit_launch(cuda_device, N, D, dtype):
    B, H = 1, 3
    q, k, v = synth.random_qkv(B, N, H, D, dtype, seed=9300 + N + D)
    scale = 1.0 / math.sqrt(D)
    ref, lse_ref = oracle.attention_ext(q, k, v, scale, dtype)
    split, lse_s = run_ext(q, k, v, scale, dtype, FORCE_ONE_TILE | SPLIT_FROM_TWO)
    whole, lse_w = run_ext(q, k, v, scale, dtype, FORCE_ONE_TILE | NO_SPLIT)
    close(split, ref, f"split N={N} D={D}")
    close(whole, ref, f"unsplit N={N} D={D}")
    close(split, whole, f"split vs unsplit N={N} D={D}")
    assert np.max(np.abs(lse_s - lse_ref)) <= 1e-3
    assert np.max(np.abs(lse_s - lse_w)) <= 1e-3


@pytest.mark.parametrize("Lq,Lk", [(200, 1000), (1000, 130), (300, 257)])
def test_split_with_cross_lengths(cuda_device, Lq, Lk):
    """More or fewer keys than queries: the halves split the key blocks of Lk."""
    rng = np.random.Generator(np.random.PCG64(9400 + Lq + Lk))
    mk = lambda n: synth.round_to_bits(rng.standard_normal((2, n, 2, 64), dtype=np.float32), synth.BF16)
    q, k, v = mk(Lq), mk(Lk), mk(Lk)
    ref, lse_ref = oracle.attention_ext(q, k, v, 0.125, synth.BF16)
    got, lse = run_ext(q, k, v, 0.125, synth.BF16, FORCE_ONE_TILE | SPLIT_FROM_TWO)
    close(got, ref, f"split Lq={Lq} Lk={Lk}")
    assert np.max(np.abs(lse - lse_ref)) <= 1e-3


def test_split_peaky_rows_merge_across_halves(cuda_device):
    """Rows whose largest logits sit in different halves for different rows
    (a scale that puts each row's maximum far above the rest), so that the
    merge must rescale either half by up to 2^-100.  V stays N(0, 1), so the
    outputs stay below 8, where a bf16 half-ulp is within the bound."""
    B, N, H, D = 1, 1024, 2, 64
    q, k, _ = synth.random_qkv(B, N, H, D, synth.BF16, seed=9500, std=3.0)
    _, _, v = synth.random_qkv(B, N, H, D, synth.BF16, seed=9501)
    ref, lse_ref = oracle.attention_ext(q, k, v, 0.5, synth.BF16)
    got, lse = run_ext(q, k, v, 0.5, synth.BF16, FORCE_ONE_TILE | SPLIT_FROM_TWO)
    close(got, ref, "peaky split")
    assert np.max(np.abs(lse - lse_ref)) <= 1e-3


def test_split_grouped_query_heads(cuda_device):
    """Grouped-query heads on a grid small enough to split."""
    import torch

    B, N, H, Hkv, D = 1, 600, 8, 2, 64
    rng = np.random.Generator(np.random.PCG64(9550))
    q = synth.round_to_bits(rng.standard_normal((B, N, H, D), dtype=np.float32), synth.BF16)
    k = synth.round_to_bits(rng.standard_normal((B, N, Hkv, D), dtype=np.float32), synth.BF16)
    v = synth.round_to_bits(rng.standard_normal((B, N, Hkv, D), dtype=np.float32), synth.BF16)
    tq, tk, tv = (to_dev(x, synth.BF16) for x in (q, k, v))
    out = torch.empty_like(tq)
    rc = vitattn.forward_gqa_ptr(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), out.data_ptr(), B, N, H, Hkv, D,
                                 0.125, synth.BF16, torch.cuda.current_stream().cuda_stream, checked=True)
    assert rc == 0, vitattn.strerror(rc)
    close(from_dev(out, synth.BF16), oracle.attention_gqa(q, k, v, 0.125, synth.BF16), "split gqa")


def test_default_launch_of_the_document_page_is_split_and_deterministic(cuda_device):
    """The document page (1 x 912 x 16 x 80) runs split by default; two
    calls give the same bits, and sampled rows match the oracle."""
    import torch

    w = synth.WORKLOADS["doc_page"]
    q, k, v = synth.make_qkv(w)
    tq, tk, tv = (to_dev(x, w.dtype) for x in (q, k, v))
    a = vitattn.forward(tq, tk, tv, scale=w.scale, checked=True)
    b = vitattn.forward(tq, tk, tv, scale=w.scale, checked=True)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    got = from_dev(a, w.dtype)
    unsplit, _ = run_ext(q, k, v, w.scale, w.dtype, NO_SPLIT, want_lse=False)
    assert not np.array_equal(got, unsplit)  # the default launch really is the split one
    ref = oracle.attention(q, k, v, w.scale, w.dtype)
    close(got, ref, "doc_page split")
