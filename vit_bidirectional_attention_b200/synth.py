"""Seeded synthetic attention inputs: the one module both the oracle and the
CUDA path are fed from.

It holds no attention arithmetic.  It draws Q, K, V as IEEE single-precision
normals from a seeded PCG64 stream, shapes them as the workloads below
describe, and rounds them once (round-to-nearest-even) to the storage dtype.
The result is a set of uint16 bit patterns that the oracle widens exactly to
double and that the GPU library reads as bf16 / f16.

Workloads (token-major ``[B, N, H, D]`` as they leave a ViT's QKV linear):

- ``tiny``       1 x 64 x 2 x 64, bf16, iid N(0,1)
- ``small_vit``  1 x 196 x 16 x 72, f16, iid N(0,1)  (14x14 patches, hidden 1152;
  the SigLIP/Gemma-4V block shape of hf2q ``vit_gpu.rs``)
- ``doc_page``   1 x 912 x 16 x 80, bf16, Q,K iid N(0, 1.5^2), V iid N(0,1)
  (the 912-patch page of inferencelayer ``vision_gpu.rs``, module doc)
- ``batched``    32 x 1024 x 16 x 64, bf16, iid N(0,1)
- ``batched_gqa`` 32 x 1024 x 16 x 64, bf16, iid N(0,1), with 4 key/value heads
  (k, v are 32 x 1024 x 4 x 64): query head h uses kv head h // 4, the
  grouped-query ratio of the Gemma-4V vision tower on the hf2q page
- ``batched_causal`` 32 x 1024 x 16 x 64, bf16, iid N(0,1), with the aligned causal
  mask (query i sees keys j <= i) and the log-sum-exp output; flops count the
  N(N+1)/2 admitted query-key pairs
- ``high_res``   2 x 16384 x 16 x 128, bf16, Q = Zq + a*Uq*W, K = Zk + a*Uk*W
  with Z iid N(0,1), U: N x 8 iid N(0,1) per tensor and per (b, h), W: 8 x D
  with orthonormal rows per (b, h) shared by Q and K, and a = sqrt(sqrt(241)-1)
  so that a logit q.k/sqrt(D) has variance 1 + (16a^2 + 8a^4)/D = 16 (std 4:
  a peaky softmax that keeps raising the running maximum); V iid N(0,1).

Ragged batches (several images' tokens packed along one axis, ``[total, H, D]``
with ``cu_seqlens`` start offsets, each image attending only within itself):

- ``multi_image``  20 images of 1024, 576, 256, 912, 196, 4096, 729, 1600, 2304,
  400, 784, 1369, 3136, 64, 2025, 900, 1156, 484, 2601 and 324 patches
  (24 936 tokens: square patch grids from 8^2 to 64^2 and the 912-patch
  page, the mixed resolutions a dynamic-resolution ViT sees; 243 MiB of
  inputs and output, more than the 126 MiB L2), 16 heads, D = 80, bf16,
  Q,K iid N(0, 1.5^2), V iid N(0,1) (the ``doc_page`` distribution).

The attention's prologue (packed QKV split + 2-D rope, ``[T, 3, H, D]`` in):

- ``rope_batched``  the QKV of ``batched``: 32 images of 32 x 32 patches
  (32 768 tokens), 16 heads, D = 64, bf16, iid N(0,1), with the 2-D rope
  tables of a 32 x 32 patch grid (``rope_tables_2d``) repeated per image.

Every workload uses scale = 1/sqrt(D) and seed 20261202 + its index.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

BF16, F16 = 0, 1
DTYPE_NAMES = {BF16: "bf16", F16: "f16"}
SEED_BASE = 20261202


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    N: int
    H: int
    D: int
    dtype: int
    qk_std: float = 1.0
    rank8_logit_std: float = 0.0  # 0: iid; >0: shared rank-8 component reaching this logit std
    index: int = 0
    Hkv: int = 0  # key/value heads (grouped-query attention); 0: as many as query heads
    causal: bool = False  # aligned causal mask (query i sees keys j <= i), with the LSE output

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def seed(self) -> int:
        return SEED_BASE + self.index

    @property
    def flops(self) -> float:
        """4*B*H*N^2*D: the two contractions QK^T and PV, two flops per MAC
        (with the causal mask only the N(N+1)/2 query-key pairs it admits)."""
        pairs = self.N * (self.N + 1) / 2 if self.causal else self.N * self.N
        return 4.0 * self.B * self.H * pairs * self.D

    @property
    def kv_heads(self) -> int:
        return self.Hkv or self.H

    @property
    def io_bytes(self) -> int:
        """Q, K, V read once and O written once, 2 bytes per element."""
        return (2 * self.H + 2 * self.kv_heads) * self.B * self.N * self.D * 2

    @property
    def numel(self) -> int:
        return self.B * self.N * self.H * self.D


WORKLOADS = {
    w.name: w
    for w in (
        Workload("tiny", 1, 64, 2, 64, BF16, index=0),
        Workload("small_vit", 1, 196, 16, 72, F16, index=1),
        Workload("doc_page", 1, 912, 16, 80, BF16, qk_std=1.5, index=2),
        Workload("batched", 32, 1024, 16, 64, BF16, index=3),
        Workload("high_res", 2, 16384, 16, 128, BF16, rank8_logit_std=4.0, index=4),
        # the batched shape with 4 query heads per key/value head (the GQA ratio of the
        # Gemma-4V vision tower on the hf2q page)
        Workload("batched_gqa", 32, 1024, 16, 64, BF16, index=7, Hkv=4),
        # the batched shape with the aligned causal mask and the LSE output
        Workload("batched_causal", 32, 1024, 16, 64, BF16, index=8, causal=True),
    )
}


@dataclasses.dataclass(frozen=True)
class RaggedWorkload:
    name: str
    seqlens: tuple
    H: int
    D: int
    dtype: int
    qk_std: float = 1.0
    index: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def seed(self) -> int:
        return SEED_BASE + self.index

    @property
    def cu_seqlens(self) -> list:
        cu = [0]
        for n in self.seqlens:
            cu.append(cu[-1] + n)
        return cu

    @property
    def total(self) -> int:
        return sum(self.seqlens)

    @property
    def flops(self) -> float:
        """4*H*D*sum(n_s^2): each image's QK^T and PV, two flops per MAC."""
        return 4.0 * self.H * self.D * sum(n * n for n in self.seqlens)

    @property
    def io_bytes(self) -> int:
        return 4 * self.total * self.H * self.D * 2

    @property
    def numel(self) -> int:
        return self.total * self.H * self.D


RAGGED = {
    w.name: w
    for w in (
        RaggedWorkload("multi_image", (1024, 576, 256, 912, 196, 4096, 729, 1600, 2304, 400,
                                       784, 1369, 3136, 64, 2025, 900, 1156, 484, 2601, 324), 16, 80, BF16,
                       qk_std=1.5, index=5),
    )
}


def make_qkv_ragged(w: RaggedWorkload, seed: int | None = None):
    """(q, k, v) uint16 bit arrays of shape [total, H, D] for ragged workload ``w``."""
    rng = np.random.Generator(np.random.PCG64(w.seed if seed is None else seed))
    shape = (w.total, w.H, w.D)
    out = []
    for std in (w.qk_std, w.qk_std, 1.0):
        x = rng.standard_normal(size=shape, dtype=np.float32)
        if std != 1.0:
            x *= np.float32(std)
        out.append(round_to_bits(x, w.dtype))
    return tuple(out)


def random_ragged(seqlens, H: int, D: int, dtype: int, seed: int, std: float = 1.0):
    """iid N(0, std^2) ragged inputs ``[total, H, D]`` and their cu_seqlens."""
    w = RaggedWorkload("sweep", tuple(int(n) for n in seqlens), H, D, dtype, qk_std=std)
    q, k, v = make_qkv_ragged(w, seed=seed)
    return q, k, v, w.cu_seqlens


def rope_tables_2d(grid_h: int, grid_w: int, D: int, theta: float = 10000.0):
    """cos, sin ``[grid_h*grid_w, D]`` float32 for the patches of an h x w grid
    in row-major order: a 2-D rotary embedding whose first D/4 frequency pairs
    turn with the patch row and the next D/4 with the patch column, each
    angle shared by the pair (d, d + D/2) that ``rotate_half`` rotates.
    (These are the kernel's inputs, built the way the pages say the CPU
    tower builds them: a (row, col) walk, with the rotation applied
    elsewhere.)"""
    quarter = D // 4
    inv_freq = theta ** (-np.arange(quarter, dtype=np.float64) / quarter)
    r, c = np.divmod(np.arange(grid_h * grid_w, dtype=np.float64), grid_w)
    ang = np.concatenate([r[:, None] * inv_freq[None, :], c[:, None] * inv_freq[None, :]], axis=1)
    if ang.shape[1] < D // 2:  # D/2 odd: the last pair gets angle 0
        ang = np.concatenate([ang, np.zeros((ang.shape[0], D // 2 - ang.shape[1]))], axis=1)
    ang = np.concatenate([ang, ang], axis=1)
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


@dataclasses.dataclass(frozen=True)
class PrologueWorkload:
    """A packed QKV projection of ``images`` images of ``grid`` patches each,
    with their 2-D rope tables: the input of the QKV split + rope prologue."""
    name: str
    images: int
    grid: tuple
    H: int
    D: int
    dtype: int
    index: int = 0
    qk_norm: bool = False   # per-head RMS norm of q and k before the rope
    eps: float = 1e-6

    @property
    def seed(self) -> int:
        return SEED_BASE + self.index

    @property
    def T(self) -> int:
        return self.images * self.grid[0] * self.grid[1]

    @property
    def io_bytes(self) -> int:
        """qkv read, cos/sin read, q/k/v written: each once (plus the two
        [D] f32 norm weights when ``qk_norm``)."""
        return 2 * (3 * self.T * self.H * self.D * 2) + 2 * self.T * self.D * 4 + (8 * self.D if self.qk_norm else 0)


PROLOGUE = {
    w.name: w
    for w in (
        # the QKV of the batched workload: 32 images of 32 x 32 patches, 16 heads, D = 64
        PrologueWorkload("rope_batched", 32, (32, 32), 16, 64, BF16, index=6),
        # the same, with the q/k RMS norm ahead of the rope (the GLM-OCR tower's prologue)
        PrologueWorkload("rope_norm_batched", 32, (32, 32), 16, 64, BF16, index=9, qk_norm=True),
    )
}


@dataclasses.dataclass(frozen=True)
class LayerWorkload:
    """The attention step of one ViT layer from its packed QKV projection:
    the prologue (split + 2-D rope) and the attention, on ``images`` images
    of ``grid`` patches.  ``packed``: the q/k-only prologue and the attention
    reading v straight from the projection (token stride 3*H*D); otherwise
    the full prologue (which copies v) and the dense attention."""
    name: str
    images: int
    grid: tuple
    H: int
    D: int
    dtype: int
    packed: bool
    index: int = 0

    @property
    def seed(self) -> int:
        return SEED_BASE + self.index

    @property
    def N(self) -> int:
        return self.grid[0] * self.grid[1]

    @property
    def T(self) -> int:
        return self.images * self.N

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def flops(self) -> float:
        return 4.0 * self.images * self.H * self.N * self.N * self.D

    @property
    def prologue_bytes(self) -> int:
        """The prologue's reads and writes: q and k (and v unless packed) in
        and out once, plus the two f32 rope tables."""
        parts = 2 if self.packed else 3
        return 2 * parts * self.T * self.H * self.D * 2 + 2 * self.T * self.D * 4

    @property
    def attention_bytes(self) -> int:
        """q, k, v read once and the output written once."""
        return 4 * self.T * self.H * self.D * 2

    @property
    def io_bytes(self) -> int:
        return self.prologue_bytes + self.attention_bytes


LAYER = {
    w.name: w
    for w in (
        # the batched workload's layer (32 images of 32 x 32 patches, 16 heads, D = 64)
        LayerWorkload("layer_batched", 32, (32, 32), 16, 64, BF16, packed=False, index=6),
        LayerWorkload("layer_packed_batched", 32, (32, 32), 16, 64, BF16, packed=True, index=6),
    )
}


def make_prologue(w: PrologueWorkload):
    """(qkv bits [T, 3, H, D], cos [T, D], sin [T, D]) for prologue workload ``w``."""
    qkv = make_qkv_packed(w.T, w.H, w.D, w.dtype, seed=w.seed)
    cs, sn = rope_tables_2d(w.grid[0], w.grid[1], w.D)
    return qkv, np.tile(cs, (w.images, 1)), np.tile(sn, (w.images, 1))


def make_norm_weights(D: int, seed: int):
    """(q_norm_w, k_norm_w) float32 ``[D]`` each: 1 + 0.25 * N(0, 1), the
    spread of a trained RMS-norm weight around its initial value of one."""
    rng = np.random.Generator(np.random.PCG64(seed))
    w = 1.0 + 0.25 * rng.standard_normal(size=(2, D))
    return w[0].astype(np.float32), w[1].astype(np.float32)


def make_qkv_packed(T: int, H: int, D: int, dtype: int, seed: int, std: float = 1.0):
    """A packed QKV projection output ``[T, 3, H, D]`` (bit patterns), iid N(0, std^2)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal(size=(T, 3, H, D), dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return round_to_bits(x, dtype)


def round_to_bits(x: np.ndarray, dtype: int) -> np.ndarray:
    """float32 -> bf16 / f16 bit patterns, round to nearest even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == F16:
        return x.astype(np.float16).view(np.uint16)
    if dtype != BF16:
        raise ValueError(f"unknown dtype code {dtype}")
    u = x.view(np.uint32).astype(np.uint64)
    nan = (u & 0x7F800000) == 0x7F800000
    nan &= (u & 0x007FFFFF) != 0
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    rounded = np.where(nan, (u >> 16) | 0x40, rounded)
    return rounded.astype(np.uint16)


def bits_to_float32(bits: np.ndarray, dtype: int) -> np.ndarray:
    """Inverse of :func:`round_to_bits` (exact)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    if dtype == F16:
        return bits.view(np.float16).astype(np.float32)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _rank8_alpha(D: int, logit_std: float) -> float:
    # logit variance 1 + (16 a^2 + 8 a^4) / D = logit_std^2  ->  a^4 + 2 a^2 - c = 0
    c = (logit_std * logit_std - 1.0) * D / 8.0
    a2 = -1.0 + math.sqrt(1.0 + c)
    return math.sqrt(a2)


def make_qkv(w: Workload, seed: int | None = None):
    """(q, k, v) uint16 bit arrays of shape [B, N, H, D] for workload ``w``."""
    rng = np.random.Generator(np.random.PCG64(w.seed if seed is None else seed))
    shape = (w.B, w.N, w.H, w.D)
    if w.Hkv:
        kv_shape = (w.B, w.N, w.Hkv, w.D)
        q = rng.standard_normal(size=shape, dtype=np.float32) * np.float32(w.qk_std)
        k = rng.standard_normal(size=kv_shape, dtype=np.float32) * np.float32(w.qk_std)
        v = rng.standard_normal(size=kv_shape, dtype=np.float32)
        return tuple(round_to_bits(x, w.dtype) for x in (q, k, v))

    def normal(std: float = 1.0) -> np.ndarray:
        x = rng.standard_normal(size=shape, dtype=np.float32)
        if std != 1.0:
            x *= np.float32(std)
        return x

    if w.rank8_logit_std > 0.0:
        alpha = np.float32(_rank8_alpha(w.D, w.rank8_logit_std))
        zq = normal()
        zk = normal()
        for b in range(w.B):
            for h in range(w.H):
                g = rng.standard_normal(size=(w.D, 8))
                basis, _ = np.linalg.qr(g)                     # D x 8, orthonormal columns
                W = basis.T.astype(np.float32)                 # 8 x D, orthonormal rows
                uq = rng.standard_normal(size=(w.N, 8), dtype=np.float32)
                uk = rng.standard_normal(size=(w.N, 8), dtype=np.float32)
                zq[b, :, h, :] += alpha * (uq @ W)
                zk[b, :, h, :] += alpha * (uk @ W)
        q, k = zq, zk
    else:
        q = normal(w.qk_std)
        k = normal(w.qk_std)
    v = normal()
    return tuple(round_to_bits(x, w.dtype) for x in (q, k, v))


def random_qkv(B: int, N: int, H: int, D: int, dtype: int, seed: int, std: float = 1.0):
    """iid N(0, std^2) inputs for shape sweeps (same recipe, free shape)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    out = []
    for _ in range(3):
        x = rng.standard_normal(size=(B, N, H, D), dtype=np.float32)
        if std != 1.0:
            x *= np.float32(std)
        out.append(round_to_bits(x, dtype))
    return tuple(out)


def sample_rows(w_or_shape, count: int, seed: int) -> np.ndarray:
    """``count`` distinct flat token-head row indices ``(b*N + i)*H + h``,
    always including the first and last row of the tensor."""
    if isinstance(w_or_shape, Workload):
        B, N, H = w_or_shape.B, w_or_shape.N, w_or_shape.H
    else:
        B, N, H = w_or_shape[:3]
    total = B * N * H
    count = min(count, total)
    rng = np.random.Generator(np.random.PCG64(seed))
    rows = rng.choice(total, size=count, replace=False).astype(np.int64)
    rows[0] = 0
    if count > 1:
        rows[-1] = total - 1
    return np.unique(rows)
