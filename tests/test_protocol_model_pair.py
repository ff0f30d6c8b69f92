"""The planned paired-CTA barrier protocol (``tests/protocol_model_pair.py``),
replayed on the CPU under random schedules before any kernel implements it:
for one or two query tiles per CTA, two or three S buffers, one or two Q
buffers, looping or not, bf16 or f16 and a 4- or 8-slot K/V ring, no parity
wait may pass on the wrong phase, no arrival may land in another phase,
and nothing may deadlock.  Planted mistakes must be caught."""
import inspect
import itertools
import types

import pytest

import protocol_model_pair
from protocol_model_pair import run_pair

CONFIGS = [
    (T, NS, NQ, loop, bf16, KS)
    for T, NS, NQ, loop, bf16, KS in itertools.product([1, 2], [2, 3], [1, 2], [False, True], [False, True], [4, 8])
    if loop or NQ == 1
]


@pytest.mark.parametrize("T,NS,NQ,loop,bf16,KS", CONFIGS)
def test_paired_protocol_has_no_aliasing_stray_arrival_or_deadlock(T, NS, NQ, loop, bf16, KS):
    for nkb in (1, 2, 3, 5, 8):
        for n_my in ((1, 2, 3) if loop else (1,)):
            for seed in range(6):
                run_pair(T, NS, NQ, nkb, n_my, loop, bf16, seed, KS)


def mutant(replacements):
    text = inspect.getsource(protocol_model_pair)
    for a, b in replacements:
        assert a in text, a
        text = text.replace(a, b)
    mod = types.ModuleType("protocol_model_pair_mutant")
    exec(compile(text, "protocol_model_pair_mutant", "exec"), mod.__dict__)
    return mod


def failures(mod, args, seeds=200):
    n = 0
    for seed in range(seeds):
        try:
            mod.run_pair(*args[:7], seed, *args[7:])
        except AssertionError:
            n += 1
    return n


def test_one_p_written_barrier_per_tile_is_caught():
    """With a single shared "P written" barrier per tile, one CTA's softmax can
    arrive for a later block while the other CTA's arrival for the current
    block is still missing."""
    mod = mutant([('("wait", ("p_full", t, g & 1), g >> 1)', '("wait", ("p_full", t, 0), g)'),
                  ('("arrive", ("p_full", t, g & 1), 128, g >> 1)', '("arrive", ("p_full", t, 0), 128, g)')])
    assert failures(mod, (2, 3, 1, 8, 1, False, True)) > 0


def test_a_commit_to_the_leader_only_is_caught():
    """If the MMA's S-ready commit reached only the leader, the follower's
    softmax would wait forever."""
    mod = mutant([('commits = [(n, u // ns) for n in both("s_full", buf)]',
                   'commits = [(("s_full", 0, buf), u // ns)]')])
    assert failures(mod, (2, 3, 1, 3, 1, False, False), seeds=20) == 20


def test_a_converter_waiting_on_the_gathering_barrier_is_caught():
    """A bf16 converter that waited on the leader's K/V barrier, instead of its
    own CTA's V-landed barrier, would never see the V halves (they signal
    ``v_landed``): the model reports the deadlock."""
    mod = mutant([('yield ("wait", ("v_landed", c, idx % KS), idx // KS)',
                   'yield ("wait", ("kv_full", idx % KS), idx // KS)')])
    assert failures(mod, (1, 2, 1, 3, 1, False, True), seeds=20) == 20
