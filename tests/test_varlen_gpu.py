"""GPU parity for ragged multi-image batches: the CUDA path through the C ABI
(``vitattn_forward_varlen``) against the fp64 oracle's ``attention_varlen``.

Several images' tokens are packed along one axis, ``[total, H, D]``, with
start offsets ``cu_seqlens``; each token attends only to its own image
(inferencelayer ``src/vision_gpu.rs``, the vision tower's ``forward``:
attention over an image is one ragged segment, several images are several
segments).  Tolerance as for the dense path: max |O_gpu - O_ref| <= 1e-2 and
||O_gpu - O_ref||_F / ||O_ref||_F <= 4e-3.
"""
import numpy as np
import pytest

import oracle
from vit_bidirectional_attention_b200 import synth, vitattn

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
REL_FROB = 4e-3
FORCE_TWO_TILES = 2
FORCE_ONE_TILE = 4
NO_SPLIT = 16  # ragged batches never split a tile's key blocks; keep the dense call alike


def to_dev(bits, dtype):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy())
    return t.view(torch.bfloat16 if dtype == synth.BF16 else torch.float16).cuda()


def from_dev(t, dtype):
    import torch

    return synth.bits_to_float32(t.view(torch.int16).cpu().numpy().view(np.uint16), dtype).astype(np.float64)


def run_varlen(q, k, v, cu, scale, dtype, flags=0):
    import torch

    tq, tk, tv = (to_dev(x, dtype) for x in (q, k, v))
    out = torch.full_like(tq, float("nan"))
    _, H, D = q.shape
    rc = vitattn.forward_varlen_ptr(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), out.data_ptr(), cu, H, D, scale,
                                    dtype, torch.cuda.current_stream().cuda_stream, checked=True, flags=flags)
    assert rc == 0, vitattn.strerror(rc)
    return from_dev(out, dtype)


def assert_close(got, ref, what=""):
    assert np.all(np.isfinite(got)), f"{what}: non-finite output (a token left unwritten?)"
    max_abs = float(np.max(np.abs(got - ref)))
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    assert max_abs <= MAX_ABS and rel <= REL_FROB, f"{what}: max_abs={max_abs:.3e} rel_frob={rel:.3e}"


MIXES = [
    [1],
    [64, 196, 1],
    [129, 127, 256, 0, 300],
    [0, 0, 5, 0],
    [255, 257, 128, 384, 513],
    [1024, 77, 912],
]


@pytest.mark.parametrize("tiles", [FORCE_TWO_TILES, FORCE_ONE_TILE])
@pytest.mark.parametrize("mix", range(len(MIXES)))
@pytest.mark.parametrize("D,dtype", [(64, synth.BF16), (80, synth.BF16), (128, synth.F16), (16, synth.F16)])
def test_segment_mixes(cuda_device, mix, D, dtype, tiles):
    q, k, v, cu = synth.random_ragged(MIXES[mix], 3, D, dtype, seed=7000 + 31 * mix + D + dtype, std=1.3)
    scale = 1.0 / np.sqrt(D)
    got = run_varlen(q, k, v, cu, scale, dtype, flags=tiles)
    assert_close(got, oracle.attention_varlen(q, k, v, cu, scale, dtype), f"mix {MIXES[mix]} D={D} flags {tiles}")


def test_multi_image_workload_full_parity(cuda_device):
    """The benchmarked ragged workload (20 images, 24 936 tokens), every output element."""
    w = synth.RAGGED["multi_image"]
    q, k, v = synth.make_qkv_ragged(w)
    got = run_varlen(q, k, v, w.cu_seqlens, w.scale, w.dtype)
    assert_close(got, oracle.attention_varlen(q, k, v, w.cu_seqlens, w.scale, w.dtype), "multi_image")


def test_many_short_segments(cuda_device):
    lens = np.random.Generator(np.random.PCG64(7100)).integers(0, 40, size=256)
    q, k, v, cu = synth.random_ragged(lens, 2, 64, synth.BF16, seed=7101)
    got = run_varlen(q, k, v, cu, 0.125, synth.BF16)
    assert_close(got, oracle.attention_varlen(q, k, v, cu, 0.125, synth.BF16), "256 segments")


@pytest.mark.parametrize("tiles", [FORCE_TWO_TILES, FORCE_ONE_TILE])
def test_equal_segments_match_the_dense_entry_bitwise(cuda_device, tiles):
    """B images of N tokens each, packed, give exactly what the dense [B, N, H, D]
    call gives: keys past an image are masked to probability 0 in both (the
    dense call with its key blocks unsplit, as ragged batches run)."""
    import torch

    B, N, H, D = 3, 300, 2, 64
    q, k, v = synth.random_qkv(B, N, H, D, synth.BF16, seed=7200)
    tq, tk, tv = (to_dev(x, synth.BF16) for x in (q, k, v))
    dense = torch.empty_like(tq)
    rc = vitattn.forward_ptr(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), dense.data_ptr(), B, N, H, D, 0.125,
                             synth.BF16, torch.cuda.current_stream().cuda_stream, flags=tiles | NO_SPLIT)
    assert rc == 0
    packed = run_varlen(q.reshape(B * N, H, D), k.reshape(B * N, H, D), v.reshape(B * N, H, D),
                        [0, N, 2 * N, 3 * N], 0.125, synth.BF16, flags=tiles)
    assert np.array_equal(packed.reshape(B, N, H, D), from_dev(dense, synth.BF16))


def test_images_do_not_see_each_other(cuda_device):
    cu = [0, 200, 530, 700]
    q, k, v, _ = synth.random_ragged([200, 330, 170], 2, 80, synth.BF16, seed=7300)
    a = run_varlen(q, k, v, cu, 0.11, synth.BF16)
    k2, v2 = k.copy(), v.copy()
    k2[200:530], v2[200:530] = k2[200:530][::-1], v2[200:530][:, ::-1]  # change image 1 only
    b = run_varlen(q, k2, v2, cu, 0.11, synth.BF16)
    assert np.array_equal(a[:200], b[:200]) and np.array_equal(a[530:], b[530:])
    assert not np.array_equal(a[200:530], b[200:530])


def test_bad_offsets_are_rejected_before_launch(cuda_device):
    import torch

    t = torch.zeros((100, 2, 64), dtype=torch.bfloat16, device="cuda")
    o = torch.zeros_like(t)
    with pytest.raises(vitattn.VitAttnError) as e:
        vitattn.forward_varlen(t, t, t, [0, 60, 50, 100], out=o)
    assert e.value.status == -12
    with pytest.raises(ValueError):
        vitattn.forward_varlen(t, t, t, [0, 60, 99], out=o)


def test_python_entry_on_a_side_stream(cuda_device):
    import torch

    q, k, v, cu = synth.random_ragged([100, 333], 4, 72, synth.F16, seed=7400)
    tq, tk, tv = (to_dev(x, synth.F16) for x in (q, k, v))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out = vitattn.forward_varlen(tq, tk, tv, cu, stream=s)
    s.synchronize()
    assert_close(from_dev(out, synth.F16), oracle.attention_varlen(q, k, v, cu, 1.0 / np.sqrt(72), synth.F16))
