"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Tolerance for every floating-point comparison: max |O_gpu - O_ref| <= 1e-2
and ||O_gpu - O_ref||_F / ||O_ref||_F <= 4e-3, with O_ref the oracle on the
same bf16/f16-rounded inputs.  The operation is O = softmax(scale Q K^T) V
per (batch, head), no mask (hf2q ``src/inference/vision/vit_gpu.rs``, doc of
``vit_attention_gpu``).
"""
import math

import numpy as np
import pytest

import oracle
from vit_bidirectional_attention_b200 import synth, vitattn

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
REL_FROB = 4e-3


def torch_dtype(dtype):
    import torch

    return torch.bfloat16 if dtype == synth.BF16 else torch.float16


def to_dev(bits, dtype):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy())
    return t.view(torch_dtype(dtype)).cuda()


def from_dev(t, dtype):
    import torch

    bits = t.view(torch.int16).cpu().numpy().view(np.uint16)
    return synth.bits_to_float32(bits, dtype).astype(np.float64)


FORCE_TWO_TILES = 2
FORCE_ONE_TILE = 4
TINY_GRID = 8


def run_gpu(q, k, v, scale, dtype, flags=0):
    import torch

    tq, tk, tv = (to_dev(x, dtype) for x in (q, k, v))
    if not flags:
        out = vitattn.forward(tq, tk, tv, scale=scale, checked=True)
        return from_dev(out, dtype)
    B, N, H, D = q.shape
    out = torch.empty_like(tq)
    rc = vitattn.forward_ptr(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), out.data_ptr(), B, N, H,
                             D, scale, dtype, torch.cuda.current_stream().cuda_stream, flags=flags)
    assert rc == 0, vitattn.strerror(rc)
    return from_dev(out, dtype)


def errors(got, ref):
    max_abs = float(np.max(np.abs(got - ref)))
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    return max_abs, rel


def assert_close(got, ref, what=""):
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    max_abs, rel = errors(got, ref)
    assert max_abs <= MAX_ABS and rel <= REL_FROB, f"{what}: max_abs={max_abs:.3e} rel_frob={rel:.3e}"


# ------------------------------------------------------------------ the workloads

@pytest.mark.parametrize("name", ["tiny", "small_vit", "doc_page"])
def test_workload_full_parity(cuda_device, name):
    w = synth.WORKLOADS[name]
    q, k, v = synth.make_qkv(w)
    got = run_gpu(q, k, v, w.scale, w.dtype)
    ref = oracle.attention(q, k, v, w.scale, w.dtype)
    assert_close(got, ref, name)


@pytest.mark.parametrize("name,rows", [("batched", 4096), ("high_res", 1536)])
def test_workload_sampled_parity_at_full_size(cuda_device, name, rows):
    """Full-size launch (the configuration the benchmark times); the oracle
    recomputes a seeded sample of output rows, first and last row included."""
    w = synth.WORKLOADS[name]
    q, k, v = synth.make_qkv(w)
    got = run_gpu(q, k, v, w.scale, w.dtype).reshape(-1, w.D)
    idx = synth.sample_rows(w, rows, seed=w.seed + 7)
    ref = oracle.attention_rows(q, k, v, w.scale, w.dtype, idx)
    assert_close(got[idx], ref, name)
    # property at any size: every row is a convex combination of V rows, so
    # each output coordinate lies inside [min_j V, max_j V] of its head
    vf = synth.bits_to_float32(v, w.dtype).astype(np.float64)
    vmin = vf.min(axis=1, keepdims=True)
    vmax = vf.max(axis=1, keepdims=True)
    g4 = got.reshape(w.B, w.N, w.H, w.D)
    tol = 1e-2
    assert np.all(g4 >= vmin - tol) and np.all(g4 <= vmax + tol)


# ------------------------------------------------------------------ shape sweep

SWEEP_N = [1, 2, 63, 64, 65, 127, 128, 129, 196, 255, 256, 257, 384, 912, 1024]


@pytest.mark.parametrize("tiles", [FORCE_TWO_TILES, FORCE_ONE_TILE])
@pytest.mark.parametrize("N", SWEEP_N)
@pytest.mark.parametrize("D", [64, 80, 128])
def test_sweep_tokens(cuda_device, N, D, tiles):
    """Ragged and exact token counts, with two query tiles per CTA (three S
    buffers at D = 64) and with one."""
    q, k, v = synth.random_qkv(1, N, 2, D, synth.BF16, seed=1000 + N * 7 + D)
    scale = 1.0 / math.sqrt(D)
    assert_close(run_gpu(q, k, v, scale, synth.BF16, flags=tiles),
                 oracle.attention(q, k, v, scale, synth.BF16), f"N={N} D={D} tiles flag {tiles}")


@pytest.mark.parametrize("tiles", [FORCE_TWO_TILES, FORCE_ONE_TILE])
@pytest.mark.parametrize("dtype", [synth.BF16, synth.F16])
@pytest.mark.parametrize("D", [16, 24, 32, 40, 48, 56, 64, 72, 80, 88, 96, 104, 112, 120, 128])
@pytest.mark.parametrize("N", [1, 129, 257])
def test_sweep_head_dims(cuda_device, dtype, D, N, tiles):
    q, k, v = synth.random_qkv(1, N, 3, D, dtype, seed=2000 + N * 131 + D * 3 + dtype)
    scale = 1.0 / math.sqrt(D)
    assert_close(run_gpu(q, k, v, scale, dtype, flags=tiles), oracle.attention(q, k, v, scale, dtype),
                 f"N={N} D={D} dtype={dtype} tiles flag {tiles}")


def test_many_batches_and_heads(cuda_device):
    q, k, v = synth.random_qkv(3, 200, 5, 72, synth.F16, seed=3001)
    assert_close(run_gpu(q, k, v, 0.1, synth.F16), oracle.attention(q, k, v, 0.1, synth.F16))


@pytest.mark.parametrize("scale", [0.0, -0.3, 1.0, 2.5])
def test_scales(cuda_device, scale):
    q, k, v = synth.random_qkv(1, 300, 2, 64, synth.BF16, seed=3002)
    assert_close(run_gpu(q, k, v, scale, synth.BF16), oracle.attention(q, k, v, scale, synth.BF16),
                 f"scale={scale}")


def test_peaky_logits_rescale_path(cuda_device):
    """Logit std ~4 (high-res recipe at reduced N): the running max keeps rising."""
    w = synth.Workload("peaky", 1, 2048, 4, 128, synth.BF16, rank8_logit_std=4.0, index=4)
    q, k, v = synth.make_qkv(w)
    assert_close(run_gpu(q, k, v, w.scale, w.dtype), oracle.attention(q, k, v, w.scale, w.dtype))


@pytest.mark.parametrize("tiles", [FORCE_TWO_TILES, FORCE_ONE_TILE])
def test_peaky_rescale_with_each_tile_mode(cuda_device, tiles):
    w = synth.Workload("peaky64", 1, 1536, 2, 64, synth.BF16, rank8_logit_std=4.0, index=4)
    q, k, v = synth.make_qkv(w)
    assert_close(run_gpu(q, k, v, w.scale, w.dtype, flags=tiles),
                 oracle.attention(q, k, v, w.scale, w.dtype), f"tiles flag {tiles}")


@pytest.mark.parametrize("tiles", [FORCE_TWO_TILES, FORCE_ONE_TILE])
@pytest.mark.parametrize("D", [64, 80, 128])
@pytest.mark.parametrize("N", [256, 768, 1000])
def test_ctas_looping_over_many_items(cuda_device, N, D, tiles):
    """At most three CTAs, each looping over many (b, h, query group) items:
    the K/V ring, the S-buffer rotation, the per-tile block counters and the
    Q buffers all carry over from item to item."""
    q, k, v = synth.random_qkv(2, N, 3, D, synth.BF16, seed=5000 + N + D + tiles)
    scale = 1.0 / math.sqrt(D)
    assert_close(run_gpu(q, k, v, scale, synth.BF16, flags=tiles | TINY_GRID),
                 oracle.attention(q, k, v, scale, synth.BF16), f"N={N} D={D} flags {tiles | TINY_GRID}")


@pytest.mark.parametrize("D", [64, 128])
def test_ctas_looping_over_items_with_rescales(cuda_device, D):
    w = synth.Workload("peaky_items", 2, 1024, 3, D, synth.BF16, rank8_logit_std=4.0, index=4)
    q, k, v = synth.make_qkv(w)
    assert_close(run_gpu(q, k, v, w.scale, w.dtype, flags=FORCE_TWO_TILES | TINY_GRID),
                 oracle.attention(q, k, v, w.scale, w.dtype))


def test_increasing_logits_force_rescale_every_block(cuda_device):
    # key j has logit ~ j/8 along q: the row max grows by ~16 per 128-key block
    N, D = 1024, 64
    q = np.zeros((1, N, 1, D), np.float32); q[..., 0] = 1.0
    k = np.zeros((1, N, 1, D), np.float32); k[0, :, 0, 0] = np.arange(N) / 8.0
    v = np.random.Generator(np.random.PCG64(3003)).standard_normal((1, N, 1, D)).astype(np.float32)
    q, k, v = (synth.round_to_bits(x, synth.BF16) for x in (q, k, v))
    assert_close(run_gpu(q, k, v, 1.0, synth.BF16), oracle.attention(q, k, v, 1.0, synth.BF16))


# ------------------------------------------------------------------ invariants on GPU output

def test_single_token_returns_v_exactly(cuda_device):
    q, k, v = synth.random_qkv(4, 1, 3, 80, synth.BF16, seed=3004)
    got = run_gpu(q, k, v, 0.11, synth.BF16)
    assert np.array_equal(got, synth.bits_to_float32(v, synth.BF16).astype(np.float64))


def test_all_ones_v(cuda_device):
    q, k, _ = synth.random_qkv(1, 700, 2, 64, synth.BF16, seed=3005, std=2.0)
    v = synth.round_to_bits(np.ones((1, 700, 2, 64), np.float32), synth.BF16)
    got = run_gpu(q, k, v, 0.125, synth.BF16)
    assert np.max(np.abs(got - 1.0)) <= MAX_ABS


def test_identical_keys_and_zero_scale_give_mean_of_v(cuda_device):
    q, k, v = synth.random_qkv(1, 333, 2, 64, synth.BF16, seed=3006)
    k = np.ascontiguousarray(np.broadcast_to(k[:, :1], k.shape))
    vf = synth.bits_to_float32(v, synth.BF16).astype(np.float64)
    mean = np.broadcast_to(vf.mean(axis=1, keepdims=True), vf.shape)
    assert_close(run_gpu(q, k, v, 0.125, synth.BF16), mean, "identical keys")
    q2, k2, _ = synth.random_qkv(1, 333, 2, 64, synth.BF16, seed=3007)
    assert_close(run_gpu(q2, k2, v, 0.0, synth.BF16), mean, "zero scale")


def test_joint_key_value_permutation(cuda_device):
    q, k, v = synth.random_qkv(1, 500, 2, 64, synth.BF16, seed=3008)
    perm = np.random.Generator(np.random.PCG64(3009)).permutation(500)
    a = run_gpu(q, k, v, 0.125, synth.BF16)
    b = run_gpu(q, np.ascontiguousarray(k[:, perm]), np.ascontiguousarray(v[:, perm]), 0.125,
                synth.BF16)
    assert_close(b, a, "permuted")


def test_bitwise_deterministic(cuda_device):
    w = synth.WORKLOADS["doc_page"]
    q, k, v = synth.make_qkv(w)
    a = run_gpu(q, k, v, w.scale, w.dtype)
    b = run_gpu(q, k, v, w.scale, w.dtype)
    assert np.array_equal(a, b)


# ------------------------------------------------------------------ entry points

def test_side_stream_and_preallocated_out(cuda_device):
    import torch

    w = synth.WORKLOADS["small_vit"]
    q, k, v = synth.make_qkv(w)
    tq, tk, tv = (to_dev(x, w.dtype) for x in (q, k, v))
    out = torch.full_like(tq, float("nan"))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        vitattn.forward(tq, tk, tv, out=out, scale=w.scale, stream=s)
    s.synchronize()
    assert_close(from_dev(out, w.dtype), oracle.attention(q, k, v, w.scale, w.dtype))


def test_host_buffer_entry_matches(cuda_device):
    import torch

    w = synth.WORKLOADS["doc_page"]
    q, k, v = synth.make_qkv(w)
    tdt = torch_dtype(w.dtype)
    hosts = [torch.from_numpy(x.view(np.int16).copy()).view(tdt).pin_memory() for x in (q, k, v)]
    hout = torch.empty_like(hosts[0]).pin_memory()
    dq, dk, dv, dout = (torch.empty(q.shape, dtype=tdt, device="cuda") for _ in range(4))
    s = torch.cuda.current_stream()
    rc = vitattn.forward_host_ptr(*(h.data_ptr() for h in hosts), hout.data_ptr(), dq.data_ptr(),
                                  dk.data_ptr(), dv.data_ptr(), dout.data_ptr(), w.B, w.N, w.H,
                                  w.D, w.scale, w.dtype, s.cuda_stream)
    assert rc == 0
    s.synchronize()
    got = from_dev(hout, w.dtype)
    assert_close(got, oracle.attention(q, k, v, w.scale, w.dtype))


@pytest.mark.parametrize("B", [9, 16])
def test_host_buffer_entry_multi_group(cuda_device, B):
    # the batch travels in groups of whole images (up to 8 groups, the last one
    # shorter when B does not divide); every image's output must match the oracle,
    # and a second call on the same buffers gives the same bits
    import torch

    q, k, v = synth.random_qkv(B, 200, 4, 64, synth.BF16, seed=31 + B)
    hosts = [torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16).pin_memory() for x in (q, k, v)]
    hout = torch.full_like(hosts[0], float("nan")).pin_memory()
    dq, dk, dv, dout = (torch.empty(q.shape, dtype=torch.bfloat16, device="cuda") for _ in range(4))
    s = torch.cuda.Stream()
    args = [h.data_ptr() for h in hosts] + [hout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                            dout.data_ptr(), B, 200, 4, 64, 0.125, synth.BF16, s.cuda_stream]
    assert vitattn.forward_host_ptr(*args) == 0
    s.synchronize()
    first = from_dev(hout, synth.BF16)
    assert_close(first, oracle.attention(q, k, v, 0.125, synth.BF16), f"B={B}")
    hout.fill_(float("nan"))
    assert vitattn.forward_host_ptr(*args) == 0
    s.synchronize()
    assert np.array_equal(from_dev(hout, synth.BF16), first)


@pytest.mark.parametrize("B,N,H,D", [(1, 300, 16, 64), (2, 700, 16, 128), (3, 257, 15, 80)])
def test_host_buffer_entry_head_groups(cuda_device, B, N, H, D):
    # fewer images than groups: each image travels as groups of heads (2-D
    # copies of the heads' columns, token-strided attention and output);
    # the output must match the oracle and, within the tolerance, the device
    # entry, and every head column of every row must be written
    import torch

    per_chunk, G, n = vitattn.host_plan(B, H, D)
    assert G > 1 and n == B * G
    q, k, v = synth.random_qkv(B, N, H, D, synth.BF16, seed=41 + N + H)
    hosts = [torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16).pin_memory() for x in (q, k, v)]
    hout = torch.full_like(hosts[0], float("nan")).pin_memory()
    dq, dk, dv, dout = (torch.empty(q.shape, dtype=torch.bfloat16, device="cuda") for _ in range(4))
    s = torch.cuda.Stream()
    args = [h.data_ptr() for h in hosts] + [hout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                            dout.data_ptr(), B, N, H, D, 1.0 / math.sqrt(D), synth.BF16, s.cuda_stream]
    assert vitattn.forward_host_ptr(*args) == 0
    s.synchronize()
    got = from_dev(hout, synth.BF16)
    assert np.all(np.isfinite(got))
    assert_close(got, oracle.attention(q, k, v, 1.0 / math.sqrt(D), synth.BF16), f"head groups {B}x{N}x{H}x{D}")
    dev = vitattn.forward(dq, dk, dv, scale=1.0 / math.sqrt(D), checked=True)
    assert_close(got, from_dev(dev, synth.BF16), "host vs device entry")


def test_host_buffer_entry_on_the_high_res_workload(cuda_device):
    """The end-to-end call the bench times on its default workload (2 x 16384
    x 16 x 128 bf16 from pinned host buffers: 16 groups of two heads, 2-D
    copies, token-strided attention): seeded output rows against the oracle,
    and every element within the tolerance (plus one bf16 ulp) of the device
    entry's output."""
    import torch

    w = synth.WORKLOADS["high_res"]
    q, k, v = synth.make_qkv(w)
    per_chunk, G, n = vitattn.host_plan(w.B, w.H, w.D)
    assert G > 1 and n == w.B * G
    tdt = torch_dtype(w.dtype)
    hosts = [torch.from_numpy(x.view(np.int16).copy()).view(tdt).pin_memory() for x in (q, k, v)]
    hout = torch.full_like(hosts[0], float("nan")).pin_memory()
    dq, dk, dv, dout = (torch.empty(q.shape, dtype=tdt, device="cuda") for _ in range(4))
    s = torch.cuda.current_stream()
    rc = vitattn.forward_host_ptr(*(h.data_ptr() for h in hosts), hout.data_ptr(), dq.data_ptr(),
                                  dk.data_ptr(), dv.data_ptr(), dout.data_ptr(), w.B, w.N, w.H,
                                  w.D, w.scale, w.dtype, s.cuda_stream)
    assert rc == 0, vitattn.strerror(rc)
    s.synchronize()
    got = synth.bits_to_float32(hout.view(torch.int16).numpy().view(np.uint16), w.dtype).astype(np.float64)
    assert np.all(np.isfinite(got))
    flat = got.reshape(-1, w.D)
    idx = synth.sample_rows(w, 512, seed=w.seed + 11)
    assert_close(flat[idx], oracle.attention_rows(q, k, v, w.scale, w.dtype, idx), "high_res host entry")
    # the device entry runs other launches (two tiles per item, no split), so
    # the two may round a value to neighbouring bf16 numbers: one ulp of
    # |x| is at most |x| * 2^-7
    dev = run_gpu(q, k, v, w.scale, w.dtype)
    assert np.all(np.abs(got - dev) <= 1e-2 + np.abs(dev) * 2.0 ** -7)
    assert np.linalg.norm(got - dev) / np.linalg.norm(dev) <= 4e-3


def test_pointers_of_host_memory_are_refused(cuda_device):
    # a plain (unregistered) host pointer passed as device memory is refused
    # before anything is enqueued, instead of reaching a tensor map
    import torch

    t = torch.zeros((1, 64, 2, 64), dtype=torch.bfloat16, device="cuda")
    o = torch.zeros_like(t)
    h = np.zeros(64 * 2 * 64 + 8, dtype=np.uint16)
    hp = (h.ctypes.data + 15) // 16 * 16
    assert vitattn.forward_ptr(hp, t.data_ptr(), t.data_ptr(), o.data_ptr(), 1, 64, 2, 64, 1.0, 0) == -10
    assert vitattn.forward_ptr(t.data_ptr(), t.data_ptr(), t.data_ptr(), hp, 1, 64, 2, 64, 1.0, 0) == -10
    torch.cuda.synchronize()


def test_errors_on_device_do_not_launch(cuda_device):
    import torch

    t = torch.zeros((1, 64, 2, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(vitattn.VitAttnError) as e:
        vitattn.forward(t, t, t, out=t)
    assert e.value.status == -6
    assert vitattn.forward_ptr(t.data_ptr() + 2, t.data_ptr(), t.data_ptr(), t.data_ptr() + 4096,
                               1, 1, 1, 64, 1.0, 0) == -5


# ------------------------------------------------------------------ f16 P.V product

def _v_in_f16_normal_range(shape, seed):
    """bf16 V with every nonzero |v| in [2^-10, 3.984375]: exact in f16, and
    still exact in f16 after scaling by 2^14 (largest |v| 65280 < 2^16)."""
    v = np.random.Generator(np.random.PCG64(seed)).standard_normal(shape).astype(np.float32)
    v = np.clip(v, -3.984375, 3.984375)
    v[np.abs(v) < 2.0 ** -10] = 0.0
    return synth.round_to_bits(v, synth.BF16)


@pytest.mark.parametrize("D", [64, 80, 128])
def test_v_scaled_to_top_of_f16_range_scales_output_exactly(cuda_device, D):
    """Scaling V by 2^14 scales every product and sum of the P.V step by a
    power of two (no rounding changes) up to |v| = 65280, the largest bf16
    value below 2^16: the output must be exactly 2^14 times the unscaled one."""
    q, k, _ = synth.random_qkv(1, 300, 2, D, synth.BF16, seed=3100 + D)
    v = _v_in_f16_normal_range(q.shape, 3101 + D)
    vf = synth.bits_to_float32(v, synth.BF16)
    v_big = synth.round_to_bits(vf * np.float32(2.0 ** 14), synth.BF16)
    assert float(np.abs(synth.bits_to_float32(v_big, synth.BF16)).max()) == 65280.0
    scale = 1.0 / math.sqrt(D)
    small = run_gpu(q, k, v, scale, synth.BF16)
    assert_close(small, oracle.attention(q, k, v, scale, synth.BF16), "unscaled")
    big = run_gpu(q, k, v_big, scale, synth.BF16)
    assert np.array_equal(big, small * 2.0 ** 14)


def test_bf16_v_outside_f16_range_is_reported(cuda_device):
    import torch

    q, k, v = synth.random_qkv(1, 200, 2, 64, synth.BF16, seed=3102)
    v = v.copy()
    v[0, 150, 1, 7] = synth.round_to_bits(np.array([70000.0], np.float32), synth.BF16)[0]
    tq, tk, tv = (to_dev(x, synth.BF16) for x in (q, k, v))
    out = torch.empty_like(tq)
    stream = torch.cuda.current_stream().cuda_stream
    rc = vitattn.forward_ptr(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), out.data_ptr(), 1, 200, 2,
                             64, 0.125, synth.BF16, stream, checked=True)
    assert rc == -11, vitattn.strerror(rc)
    # the report does not stick: an in-range call afterwards is clean and right
    _, _, v_ok = synth.random_qkv(1, 200, 2, 64, synth.BF16, seed=3103)
    assert_close(run_gpu(q, k, v_ok, 0.125, synth.BF16), oracle.attention(q, k, v_ok, 0.125, synth.BF16))


def test_bf16_v_outside_f16_range_on_the_default_entry(cuda_device):
    """The documented contract of the unchecked entry for a bf16 V value of
    magnitude >= 2^16 (here 2^17): the call returns OK; the column that value
    sits in becomes non-finite in the rows of its head (its f16 conversion
    is inf and every row gives it a nonzero weight), and every other element
    still matches the oracle.  The checked entry reports the same input as
    VITATTN_ERR_RANGE (test above)."""
    import torch

    q, k, v = synth.random_qkv(1, 200, 2, 64, synth.BF16, seed=3105)
    v = v.copy()
    v[0, 150, 1, 7] = synth.round_to_bits(np.array([2.0 ** 17], np.float32), synth.BF16)[0]
    tq, tk, tv = (to_dev(x, synth.BF16) for x in (q, k, v))
    out = torch.empty_like(tq)
    rc = vitattn.forward_ptr(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), out.data_ptr(), 1, 200, 2, 64, 0.125,
                             synth.BF16, torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    got = from_dev(out, synth.BF16)
    bad = ~np.isfinite(got)
    assert bad[0, :, 1, 7].all() and bad.sum() == 200
    ref = oracle.attention(q, k, v, 0.125, synth.BF16)
    ok = ~bad
    assert np.max(np.abs(got[ok] - ref[ok])) <= MAX_ABS


def test_f16_inputs_never_report_range(cuda_device):
    q, k, v = synth.random_qkv(1, 200, 2, 64, synth.F16, seed=3104)
    v = synth.round_to_bits(synth.bits_to_float32(v, synth.F16) * np.float32(8192.0), synth.F16)
    got = run_gpu(q, k, v, 0.125, synth.F16)
    ref = oracle.attention(q, k, v, 0.125, synth.F16)
    # relative bar: V is scaled by 2^13
    assert np.max(np.abs(got - ref)) <= MAX_ABS * 8192.0


def test_long_peaky_sequence_full_parity(cuda_device):
    """The high-resolution recipe (rank-8 logit component of std 4, D = 128) at
    N = 8192 with 6 heads, every output element against the oracle: long
    sequences of peaked rows are where the precision of P matters most."""
    w = synth.Workload("high_res_8k", 1, 8192, 6, 128, synth.BF16, rank8_logit_std=4.0, index=4)
    q, k, v = synth.make_qkv(w)
    assert_close(run_gpu(q, k, v, w.scale, w.dtype), oracle.attention(q, k, v, w.scale, w.dtype),
                 "high_res_8k")
