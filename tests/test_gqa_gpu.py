"""GPU parity for grouped-query attention (``vitattn_forward_gqa``): H query
heads share Hkv key/value heads, query head h using kv head h // (H / Hkv)
(hf2q ``src/inference/vision/vit_gpu.rs``, doc of ``vit_repeat_kv_gpu``),
against the fp64 oracle's ``attention_gqa``.  Tolerance as for the dense path.
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


def run_gqa(q, k, v, scale, dtype, flags=0):
    import torch

    tq, tk, tv = (to_dev(x, dtype) for x in (q, k, v))
    out = torch.full_like(tq, float("nan"))
    B, N, H, D = q.shape
    rc = vitattn.forward_gqa_ptr(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), out.data_ptr(), B, N, H, k.shape[2],
                                 D, scale, dtype, torch.cuda.current_stream().cuda_stream, checked=True, flags=flags)
    assert rc == 0, vitattn.strerror(rc)
    return from_dev(out, dtype)


def gqa_inputs(B, N, H, Hkv, D, dtype, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    q = synth.round_to_bits(rng.standard_normal((B, N, H, D), dtype=np.float32), dtype)
    k = synth.round_to_bits(rng.standard_normal((B, N, Hkv, D), dtype=np.float32), dtype)
    v = synth.round_to_bits(rng.standard_normal((B, N, Hkv, D), dtype=np.float32), dtype)
    return q, k, v


def assert_close(got, ref, what=""):
    assert np.all(np.isfinite(got)), what
    max_abs = float(np.max(np.abs(got - ref)))
    rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    assert max_abs <= 1e-2 and rel <= 4e-3, f"{what}: max_abs={max_abs:.3e} rel_frob={rel:.3e}"


@pytest.mark.parametrize("flags", [FORCE_TWO_TILES, FORCE_ONE_TILE, FORCE_TWO_TILES | TINY_GRID])
@pytest.mark.parametrize("H,Hkv", [(16, 4), (8, 1), (6, 2), (3, 3)])
@pytest.mark.parametrize("N,D,dtype", [(129, 64, synth.BF16), (300, 72, synth.F16), (257, 128, synth.BF16)])
def test_gqa_parity(cuda_device, N, D, dtype, H, Hkv, flags):
    q, k, v = gqa_inputs(2, N, H, Hkv, D, dtype, seed=9000 + N + D + H * 7 + Hkv)
    scale = 1.0 / math.sqrt(D)
    assert_close(run_gqa(q, k, v, scale, dtype, flags), oracle.attention_gqa(q, k, v, scale, dtype),
                 f"N={N} D={D} H={H} Hkv={Hkv} flags={flags}")


def test_gqa_with_all_heads_is_the_dense_entry_bitwise(cuda_device):
    import torch

    q, k, v = synth.random_qkv(2, 300, 4, 64, synth.BF16, seed=9100)
    got = run_gqa(q, k, v, 0.125, synth.BF16)
    tq, tk, tv = (to_dev(x, synth.BF16) for x in (q, k, v))
    dense = vitattn.forward(tq, tk, tv, scale=0.125, checked=True)
    assert np.array_equal(got, from_dev(dense, synth.BF16))


def test_gqa_workload_sampled_parity_at_full_size(cuda_device):
    w = synth.WORKLOADS["batched_gqa"]
    q, k, v = synth.make_qkv(w)
    got = run_gqa(q, k, v, w.scale, w.dtype).reshape(-1, w.D)
    rows = synth.sample_rows(w, 2048, seed=w.seed + 7)
    g = w.H // w.Hkv
    ref = oracle.attention_rows(q, np.repeat(k, g, axis=2), np.repeat(v, g, axis=2), w.scale, w.dtype, rows)
    assert_close(got[rows], ref, "batched_gqa")


def test_python_entry(cuda_device):
    q, k, v = gqa_inputs(1, 196, 16, 4, 72, synth.F16, seed=9200)
    tq, tk, tv = (to_dev(x, synth.F16) for x in (q, k, v))
    out = vitattn.forward_gqa(tq, tk, tv, checked=True)
    assert_close(from_dev(out, synth.F16), oracle.attention_gqa(q, k, v, 1.0 / math.sqrt(72), synth.F16))
