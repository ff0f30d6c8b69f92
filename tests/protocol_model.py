"""A CPU model of the attention kernel's mbarrier protocol (test
infrastructure).

The kernel (``vit_bidirectional_attention_b200/csrc/fwd_kernel.cuh``) waits
on mbarriers by phase *parity*: a wait for phase k passes when the barrier's
phase counter has moved past a phase of k's parity.  That is only right if,
whenever the wait passes, the counter stands exactly at k + 1 (one phase
completed past the one meant, not three).  This model replays the kernel's
agents -- the TMA producer, the MMA issuer (tcgen05 operations complete in
issue order, after arbitrary delays), the softmax warpgroups (a rescale, and
with it the wait for the previous P.V, happens at random), and the bf16
V converter -- under random schedules, applying exactly the kernel's parity
rule.  A softmax warpgroup runs an item's epilogue (wait for O full, release
O) after handing over the next item's first block, as the kernel does.  It
fails on

* a wait that passes while its barrier is not exactly one phase past the
  intended one (parity aliasing),
* an arrival count overflowing a phase,
* a state in which nothing can move (deadlock).

Each agent's waits, arrivals and commits follow the kernel's code, with the
phase it intends written out (the kernel passes only its parity).
"""
from __future__ import annotations

import random


class Barrier:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.ph = name, count, 0, 0

    def arrive(self, n=1):
        self.pending += n
        if self.pending > self.count:
            raise AssertionError(f"over-arrival on {self.name}")
        if self.pending == self.count:
            self.pending = 0
            self.ph += 1


def run(T, NS, NQ, nkb, n_my, loop, bf16, seed, KS=4, split=False):
    """One random schedule of one CTA: T query tiles (1 or 2), NS S buffers
    (2 or 3, as TMEM allows), NQ Q buffers, nkb key blocks per item, n_my
    items, CTAs looping over items or not, bf16 (V converter) or f16.
    split: one item whose two "tiles" are the two halves of one query tile's
    key blocks (T = 2, no loop): every unit has its own K/V pair, and the
    lower half merges the upper half's result at the end.  Returns the
    number of scheduling steps."""
    assert not split or (T == 2 and not loop and n_my == 1)
    rng = random.Random(seed)
    kbs = [nkb] * n_my  # key blocks of each item
    ns = NS if T == 2 else min(NS, 2)  # S buffers in use
    track_pv = ns != T                 # the "P.V done" barrier is committed
    VS = KS // 2                       # V slots
    bars = {}

    def B(name, count=1):
        if name not in bars:
            bars[name] = Barrier(name, count)
        return name

    for qb in range(2):
        for t in range(2):
            B(("q_full", qb, t)), B(("q_empty", qb, t))
    for s in range(KS):
        B(("kv_full", s)), B(("kv_empty", s))
    for v in range(VS):
        B(("v_ready", v), 64)
    for b in range(3):
        B(("s_full", b))
    for t in range(2):
        B(("p_full", t, 0), 128), B(("p_full", t, 1), 128)
        B(("o_ready", t)), B(("o_full", t)), B(("o_empty", t), 128)
    B(("merge",), 128)

    def loader():
        r = 0
        for k in range(n_my):
            qb = k % NQ
            for t in range(T):
                if loop and k >= NQ:
                    yield ("wait", ("q_empty", qb, t), k // NQ - 1)
                yield ("tma", ("q_full", qb, t))
            for _ in range(kbs[k] * (T if split else 1)):
                for _kv in range(2):
                    yield ("wait", ("kv_empty", r % KS), r // KS - 1)
                    yield ("tma", ("kv_full", r % KS))
                    r += 1

    def mma():
        # units in issue order: (t, j, k, g) for block j of item k, tile t
        units, g = [], 0
        for k in range(n_my):
            for j in range(kbs[k]):
                for t in range(T):
                    units.append((t, j, k, g))
                g += 1
        total = len(units)

        def unit(u):
            t, j, k, g = units[u]
            return t, j, k, g, u % ns

        def pair(t, g):  # the K/V pair a unit reads: its block's, or its own (split)
            return T * g + t if split else g

        def issue_s(u):
            t, j, k, g, buf = unit(u)
            qb = k % NQ
            if j == 0:
                yield ("wait", ("q_full", qb, t), k // NQ)
            e = pair(t, g)
            if split or t == 0:
                yield ("wait", ("kv_full", (2 * e) % KS), (2 * e) // KS)
            commits = [("s_full", buf)]
            if split or t == T - 1:
                commits.append(("kv_empty", (2 * e) % KS))
            if loop and j == kbs[k] - 1:
                commits.append(("q_empty", qb, t))
            yield ("mma", commits)

        def issue_pv(u):
            t, j, k, g, _ = unit(u)
            e = pair(t, g)
            if split or t == 0:
                if bf16:
                    yield ("wait", ("v_ready", e % VS), e // VS)
                else:
                    yield ("wait", ("kv_full", (2 * e + 1) % KS), (2 * e + 1) // KS)
            if loop and j == 0 and k > 0:
                yield ("wait", ("o_empty", t), k - 1)
            yield ("wait", ("p_full", t, g & 1), g >> 1)
            commits = []
            if track_pv:
                commits.append(("o_ready", t))
            if split or t == T - 1:
                commits.append(("kv_empty", (2 * e + 1) % KS))
            if j == kbs[k] - 1:
                commits.append(("o_full", t))
            yield ("mma", commits)

        issued = 0
        while issued < ns and issued < total:
            yield from issue_s(issued)
            issued += 1
        for s in range(total):
            yield from issue_pv(s)
            if issued < total:
                yield from issue_s(issued)
                issued += 1

    def softmax(t):
        g = 0
        o_phase = 0  # items so far with at least one block
        pend = None  # (O-full phase, has blocks) of the item whose epilogue is pending

        def finish(pending):
            phase, has_blocks = pending
            if has_blocks:
                yield ("wait", ("o_full", t), phase)
            if split:
                if t == 1:
                    yield ("arrive", ("merge",), 128)
                else:
                    yield ("wait", ("o_full", 1), 0)
                    yield ("wait", ("merge",), 0)
            if loop:
                yield ("arrive", ("o_empty", t), 128)

        for k in range(n_my):
            for j in range(kbs[k]):
                u = T * g + t
                yield ("wait", ("s_full", u % ns), u // ns)
                if j > 0 and track_pv and rng.random() < 0.5:  # a row's max grew: rescale O
                    yield ("wait", ("o_ready", t), g - 1)
                yield ("arrive", ("p_full", t, g & 1), 128)
                g += 1
                if loop and j == 0 and pend is not None:
                    yield from finish(pend)
                    pend = None
            if loop and pend is not None:  # the item had no blocks
                yield from finish(pend)
            pend = (o_phase, kbs[k] > 0)
            o_phase += kbs[k] > 0
        if pend is not None:
            yield from finish(pend)

    def converter():
        for g in range(sum(kbs) * (T if split else 1)):
            idx = 2 * g + 1
            yield ("wait", ("kv_full", idx % KS), idx // KS)
            yield ("arrive", ("v_ready", g % VS), 64)

    agents = {"load": loader(), "mma": mma()}
    for t in range(T):
        agents[f"softmax{t}"] = softmax(t)
    if bf16:
        agents["convert"] = converter()
    cur = {}
    for name, gen in agents.items():
        ev = next(gen, None)
        if ev is not None:
            cur[name] = ev
    mma_queue, tma_pending, steps = [], [], 0
    while cur or mma_queue or tma_pending:
        steps += 1
        if steps > 10 ** 6:
            raise AssertionError("no progress bound")
        runnable = []
        for name, ev in cur.items():
            if ev[0] != "wait":
                runnable.append(name)
                continue
            b, k = bars[ev[1]], ev[2]
            if k < 0:  # the phase before the first: complete by definition
                runnable.append(name)
                continue
            if (b.ph & 1) != (k & 1):  # the kernel's parity test passes
                if b.ph != k + 1:
                    raise AssertionError(f"parity aliasing: {name} waits {ev[1]} phase {k}, barrier at {b.ph}")
                runnable.append(name)
        choices = runnable + (["#mma"] if mma_queue else []) + (["#tma"] if tma_pending else [])
        if not choices:
            raise AssertionError("deadlock: " + "; ".join(f"{n} {e}" for n, e in cur.items()))
        c = rng.choice(choices)
        if c == "#mma":
            for name in mma_queue.pop(0):
                bars[name].arrive()
            continue
        if c == "#tma":
            bars[tma_pending.pop(rng.randrange(len(tma_pending)))].arrive()
            continue
        ev = cur[c]
        if ev[0] == "mma":
            mma_queue.append(ev[1])
        elif ev[0] == "tma":
            tma_pending.append(ev[1])
        elif ev[0] == "arrive":
            bars[ev[1]].arrive(ev[2])
        nxt = next(agents[c], None)
        if nxt is None:
            del cur[c]
        else:
            cur[c] = nxt
    return steps
