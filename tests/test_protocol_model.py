"""The attention kernel's barrier protocol, replayed on the CPU under random
schedules (``tests/protocol_model.py``): every configuration the kernel can
launch -- one or two query tiles, two or three S buffers, one or two Q
buffers, CTAs looping over items or not, bf16 (with the V converter) or f16 --
must never let a parity wait pass on the wrong phase and never deadlock.
Each item's epilogue runs after the next item's first block."""
import itertools

import pytest

from protocol_model import run

CONFIGS = [
    (T, NS, NQ, loop, bf16)
    for T, NS, NQ, loop, bf16 in itertools.product([1, 2], [2, 3], [1, 2], [False, True], [False, True])
    if loop or NQ == 1
]


@pytest.mark.parametrize("T,NS,NQ,loop,bf16", CONFIGS)
def test_protocol_has_no_aliasing_or_deadlock(T, NS, NQ, loop, bf16):
    for nkb in (1, 2, 3, 5, 8):
        for n_my in ((1, 2, 3) if loop else (1,)):
            for seed in range(12):
                run(T, NS, NQ, nkb, n_my, loop, bf16, seed)


@pytest.mark.parametrize("KS", [4, 6, 8])
@pytest.mark.parametrize("NS,bf16", [(2, False), (2, True), (3, False), (3, True)])
def test_split_items_have_no_aliasing_or_deadlock(NS, bf16, KS):
    """A split item: both softmax warpgroups on one query tile, each over its
    half of the key blocks with its own K/V pair per unit, merged at the
    end; with the 4-, 6- and 8-slot rings split items use."""
    for nkb in (1, 2, 3, 4, 7):
        for seed in range(16):
            run(2, NS, 1, nkb, 1, False, bf16, seed, KS=KS, split=True)


def test_the_model_catches_a_planted_mistake():
    """Sanity of the checker itself: with a single "P written" barrier per
    tile instead of one per block parity, some schedule lets a softmax run two
    phases ahead of the MMA warp, and the model reports the aliased wait."""
    import inspect
    import types

    import protocol_model

    text = inspect.getsource(protocol_model)
    mutant = text.replace('("wait", ("p_full", t, g & 1), g >> 1)', '("wait", ("p_full", t, 0), g)').replace(
        '("arrive", ("p_full", t, g & 1), 128)', '("arrive", ("p_full", t, 0), 128)')
    assert mutant != text
    mod = types.ModuleType("protocol_model_mutant")
    exec(compile(mutant, "protocol_model_mutant", "exec"), mod.__dict__)
    failures = 0
    for seed in range(200):
        try:
            mod.run(2, 3, 1, 8, 1, False, True, seed)
        except AssertionError:
            failures += 1
    assert failures > 0


def test_the_model_catches_an_epilogue_deferred_by_a_whole_item():
    """Sanity of the checker for the deferred epilogue: running item k's
    epilogue only after item k + 1 has handed over all its blocks (instead of
    its first) leaves the next P.V waiting on O-empty while the softmax waits
    on P.V -- a deadlock the model must report."""
    import inspect
    import types

    import protocol_model

    text = inspect.getsource(protocol_model)
    mutant = text.replace("if loop and j == 0 and pend is not None:", "if False:")
    assert mutant != text
    mod = types.ModuleType("protocol_model_mutant2")
    exec(compile(mutant, "protocol_model_mutant2", "exec"), mod.__dict__)
    failures = 0
    for seed in range(50):
        try:
            mod.run(1, 2, 1, 4, 3, True, False, seed)
        except AssertionError:
            failures += 1
    assert failures > 0


def test_the_model_catches_a_split_item_sharing_k_blocks():
    """Sanity of the split model: releasing a split unit's K only after the
    upper half's S (as for shared blocks) while both halves wait for their
    own K leaves the producer short of free slots -- or lets a release land
    on the wrong entry -- and the model must report it."""
    import inspect
    import types

    import protocol_model

    text = inspect.getsource(protocol_model)
    mutant = text.replace("""            if split or t == T - 1:
                commits.append(("kv_empty", (2 * e) % KS))""", """            if t == T - 1:
                commits.append(("kv_empty", (2 * e) % KS))""")
    assert mutant != text
    mod = types.ModuleType("protocol_model_mutant3")
    exec(compile(mutant, "protocol_model_mutant3", "exec"), mod.__dict__)
    failures = 0
    for seed in range(50):
        try:
            mod.run(2, 2, 1, 4, 1, False, False, seed, split=True)
        except AssertionError:
            failures += 1
    assert failures > 0
