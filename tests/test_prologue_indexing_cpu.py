"""The prologue kernels' index arithmetic, replayed on the CPU.

``qkv_rope_kernel`` and ``qkv_norm_rope_kernel`` share one mapping: a
grid-stride loop of warps over (token, group of kRopeHeadsPerWarp heads)
items, lane l holding elements 4l..4l+3 of each head row, lanes >= D/4 idle,
the rotation partner in lane l +- D/8.  This model restates that mapping
(with the launch constants read from the kernel headers) and checks, for the
shapes the tests and the bench use:
- every output element is written exactly once, and every read and write
  stays inside its buffer;
- the partner lane's element j is element d +- D/2 of the same head;
- the norm kernel's xor butterfly, over the power of two >= D/4 lanes,
  leaves every active lane with the sum of all active lanes;
- the weight-vector reads (own and partner elements) stay inside [D].
"""
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "vit_bidirectional_attention_b200", "csrc")
NUM_SMS = 148


def constant(fname, name):
    text = open(os.path.join(CSRC, fname)).read()
    m = re.search(rf"constexpr int {name} = (\d+);", text)
    assert m, f"{name} not found in {fname}"
    return int(m.group(1))


THREADS = constant("rope_kernel.cuh", "kRopeThreads")
R = constant("rope_kernel.cuh", "kRopeHeadsPerWarp")
BLOCKS_PER_SM = {"rope": 8,  # launch_rope: a grid of up to 8 blocks per SM
                 "norm": constant("norm_rope_kernel.cuh", "kNormRopeBlocksPerSm")}

SHAPES = [(1, 1, 16), (5, 3, 64), (1000, 2, 72), (333, 16, 80), (257, 4, 128), (196, 16, 72), (64, 5, 24),
          (77, 7, 64), (9, 3, 64), (32 * 1024, 16, 64)]


def warp_items(T, H, blocks_per_sm):
    """(warp id, item) pairs the grid-stride loop visits, as the host sizes the grid."""
    groups = (H + R - 1) // R
    items = T * groups
    per_block = THREADS // 32
    grid = min((items + per_block - 1) // per_block, NUM_SMS * blocks_per_sm)
    stride = grid * per_block
    seen = []
    for w in range(min(stride, items)):
        seen.append(np.arange(w, items, stride))
    return np.concatenate(seen), groups, items


@pytest.mark.parametrize("kind", ["rope", "norm"])
@pytest.mark.parametrize("T,H,D", SHAPES)
def test_every_output_element_written_once_and_reads_in_bounds(kind, T, H, D):
    it, groups, items = warp_items(T, H, BLOCKS_PER_SM[kind])
    assert np.array_equal(np.sort(it), np.arange(items))          # each item once
    t = it // groups
    h0 = (it - t * groups) * R
    nh = np.minimum(R, H - h0)
    hd2 = H * D * 2
    lanes = np.arange(D // 4)                                     # active lanes only touch memory
    writes = np.zeros(T * H * D, np.int32)
    for r in range(R):
        live = r < nh
        if not live.any():                                        # fewer than R heads in every group
            continue
        tt, hh = t[live], h0[live] + r
        in0 = tt[:, None] * 3 * hd2 + (hh[:, None] * D + 4 * lanes[None, :]) * 2
        out0 = tt[:, None] * hd2 + (hh[:, None] * D + 4 * lanes[None, :]) * 2
        for base in (in0, in0 + hd2, in0 + 2 * hd2):                # q, k, v rows of the packed input
            assert base.min() >= 0 and base.max() + 8 <= 3 * T * hd2
        assert out0.min() >= 0 and out0.max() + 8 <= T * hd2
        elem = (out0 // 2)[..., None] + np.arange(4)
        np.add.at(writes, elem.ravel(), 1)
    assert np.all(writes == 1)
    tab = t[:, None] * D + 4 * lanes[None, :]
    assert tab.min() >= 0 and tab.max() + 4 <= T * D               # cos / sin float4 reads


@pytest.mark.parametrize("D", [16, 24, 32, 48, 64, 72, 80, 96, 104, 128])
def test_partner_lane_holds_the_rotation_partner(D):
    half_lanes = D // 8
    for lane in range(D // 4):
        partner = lane + half_lanes if lane < half_lanes else lane - half_lanes
        assert 0 <= partner < D // 4
        for j in range(4):
            d = 4 * lane + j
            want = d + D // 2 if d < D // 2 else d - D // 2
            assert 4 * partner + j == want
        # the weight reads of the norm kernel: own and partner float4 inside [D]
        assert 4 * lane + 4 <= D and 4 * partner + 4 <= D


@pytest.mark.parametrize("D", [16, 24, 32, 48, 64, 72, 80, 96, 104, 128])
def test_norm_butterfly_gives_every_active_lane_the_head_sum(D):
    active = D // 4
    span = 1
    while span < active:
        span <<= 1
    rng = np.random.default_rng(D)
    own = rng.integers(1, 1 << 20, size=active)          # integers, so the sums are exact
    vals = np.zeros(32, np.int64)
    vals[:active] = own                                   # lanes in [active, span) hold zeros (loads skipped)
    vals[span:] = rng.integers(1 << 30, 1 << 31, size=32 - span)   # lanes past span: anything
    for o in (16, 8, 4, 2, 1):
        if o < span:
            vals = vals + vals[np.arange(32) ^ o]
    assert np.all(vals[:active] == int(own.sum()))


def test_launch_constants_match_the_register_budget():
    """A 256-thread block at the declared blocks per SM must fit the 65 536
    registers of an SM at the register counts the kernels compile to (56 and
    80 per thread; both checked with ptxas -v, no spills)."""
    assert THREADS == 256
    assert BLOCKS_PER_SM["norm"] * THREADS * 80 <= 65536
    assert 4 * THREADS * 56 <= 65536
