"""A CPU model of the PLANNED paired-CTA barrier protocol (test
infrastructure; no kernel implements it yet).

The planned kernel runs a cluster of two CTAs on two SMs.  The leader's MMA
warp issues M = 256 tcgen05 MMAs (``cta_group::2``) that read both CTAs'
shared memory and write both CTAs' tensor memory; each CTA keeps its own
query tiles, loads its own half of every K and V block, and runs its own
softmax over its own rows.  This model checks the barrier plan for that
design:

* barriers the leader's MMA waits on live in the leader and gather both
  CTAs: ``q_full`` and ``kv_full`` (both CTAs' TMA loads, signalled to the
  leader's barrier), ``p_full`` (256 softmax threads, the follower's by
  remote arrive), ``o_empty`` (likewise) and, for bf16, ``v_ready`` (both
  CTAs' converter warps);
* barriers the MMA completes are in both CTAs, arrived together by one
  multicast commit: ``s_full``, ``o_ready``, ``o_full``, ``kv_empty``,
  ``q_empty``;
* a CTA's bf16 converter waits on a local ``v_landed`` barrier for its own V
  half (an mbarrier can only be waited on by its own CTA).

Every wait uses the kernel's parity rule, and every arrival names the phase
it is meant for.  A run fails on
* a wait that passes while its barrier is not exactly one phase past the
  intended one;
* an arrival landing in a phase other than its own (for example, one CTA's
  softmax arriving for block g + 2 on a barrier still collecting block g);
* a state in which nothing can move.
"""
from __future__ import annotations

import random


class Barrier:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.ph = name, count, 0, 0

    def arrive(self, n, phase):
        if phase != self.ph:
            raise AssertionError(f"arrival for phase {phase} on {self.name} at phase {self.ph}")
        self.pending += n
        if self.pending > self.count:
            raise AssertionError(f"over-arrival on {self.name}")
        if self.pending == self.count:
            self.pending = 0
            self.ph += 1


def run_pair(T, NS, NQ, nkb, n_my, loop, bf16, seed, KS=8):
    """One random schedule of one CTA pair: T query tiles per CTA, NS S
    buffers per CTA, NQ Q buffers, nkb key blocks per item, n_my items, CTAs
    looping over items or not, bf16 (converter warps) or f16, KS K/V slots
    per CTA (each holding half a block).  Returns the scheduling steps."""
    rng = random.Random(seed)
    ns = NS if T == 2 else min(NS, 2)
    track_pv = ns != T
    VS = KS // 2
    bars = {}

    def B(name, count):
        bars[name] = Barrier(name, count)

    for qb in range(2):
        for t in range(2):
            B(("q_full", qb, t), 2)
            for c in range(2):
                B(("q_empty", c, qb, t), 1)
    for s in range(KS):
        B(("kv_full", s), 2)
        for c in range(2):
            B(("kv_empty", c, s), 1)
            B(("v_landed", c, s), 1)
    for v in range(VS):
        B(("v_ready", v), 128)
    for c in range(2):
        for b in range(3):
            B(("s_full", c, b), 1)
        for t in range(2):
            B(("o_ready", c, t), 1)
            B(("o_full", c, t), 1)
    for t in range(2):
        B(("p_full", t, 0), 256)
        B(("p_full", t, 1), 256)
        B(("o_empty", t), 256)

    def both(name, *rest):
        return [((name, c) + rest) for c in range(2)]

    def loader(c):
        r = 0
        for k in range(n_my):
            qb = k % NQ
            for t in range(T):
                if loop and k >= NQ:
                    yield ("wait", ("q_empty", c, qb, t), k // NQ - 1)
                yield ("tma", [(("q_full", qb, t), k // NQ)])
            for _ in range(nkb):
                for kv in range(2):  # K half, then V half
                    yield ("wait", ("kv_empty", c, r % KS), r // KS - 1)
                    if kv == 1 and bf16:
                        yield ("tma", [(("v_landed", c, r % KS), r // KS)])
                    else:
                        yield ("tma", [(("kv_full", r % KS), r // KS)])
                    r += 1

    def mma():
        total = n_my * T * nkb

        def unit(u):
            g, t = divmod(u, T)
            k, j = divmod(g, nkb)
            return t, j, k, g, u % ns

        def issue_s(u):
            t, j, k, g, buf = unit(u)
            qb = k % NQ
            if j == 0:
                yield ("wait", ("q_full", qb, t), k // NQ)
            if t == 0:
                yield ("wait", ("kv_full", (2 * g) % KS), (2 * g) // KS)
            commits = [(n, u // ns) for n in both("s_full", buf)]
            if t == T - 1:
                commits += [(n, (2 * g) // KS) for n in both("kv_empty", (2 * g) % KS)]
            if loop and j == nkb - 1:
                commits += [(n, k // NQ) for n in both("q_empty", qb, t)]
            yield ("mma", commits)

        def issue_pv(u):
            t, j, k, g, _ = unit(u)
            if t == 0:
                if bf16:
                    yield ("wait", ("v_ready", g % VS), g // VS)
                else:
                    yield ("wait", ("kv_full", (2 * g + 1) % KS), (2 * g + 1) // KS)
            if loop and j == 0 and k > 0:
                yield ("wait", ("o_empty", t), k - 1)
            yield ("wait", ("p_full", t, g & 1), g >> 1)
            commits = []
            if track_pv:
                commits += [(n, g) for n in both("o_ready", t)]
            if t == T - 1:
                commits += [(n, (2 * g + 1) // KS) for n in both("kv_empty", (2 * g + 1) % KS)]
            if j == nkb - 1:
                commits += [(n, k) for n in both("o_full", t)]
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

    def softmax(c, t):
        g = 0
        for k in range(n_my):
            for j in range(nkb):
                u = T * g + t
                yield ("wait", ("s_full", c, u % ns), u // ns)
                if j > 0 and track_pv and rng.random() < 0.5:  # a row's max grew: rescale O
                    yield ("wait", ("o_ready", c, t), g - 1)
                yield ("arrive", ("p_full", t, g & 1), 128, g >> 1)
                g += 1
            yield ("wait", ("o_full", c, t), k)
            if loop:
                yield ("arrive", ("o_empty", t), 128, k)

    def converter(c):
        for g in range(n_my * nkb):
            idx = 2 * g + 1
            yield ("wait", ("v_landed", c, idx % KS), idx // KS)
            yield ("arrive", ("v_ready", g % VS), 64, g // VS)

    agents = {"mma": mma()}
    for c in range(2):
        agents[f"load{c}"] = loader(c)
        for t in range(T):
            agents[f"softmax{c}.{t}"] = softmax(c, t)
        if bf16:
            agents[f"convert{c}"] = converter(c)
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
            if k < 0:
                runnable.append(name)
                continue
            if (b.ph & 1) != (k & 1):
                if b.ph != k + 1:
                    raise AssertionError(f"parity aliasing: {name} waits {ev[1]} phase {k}, barrier at {b.ph}")
                runnable.append(name)
        choices = runnable + (["#mma"] if mma_queue else []) + (["#tma"] if tma_pending else [])
        if not choices:
            raise AssertionError("deadlock: " + "; ".join(f"{n} {e}" for n, e in cur.items()))
        c = rng.choice(choices)
        if c == "#mma":  # tcgen05 operations complete in issue order
            for name, phase in mma_queue.pop(0):
                bars[name].arrive(1, phase)
            continue
        if c == "#tma":  # TMA loads complete in any order
            for name, phase in tma_pending.pop(rng.randrange(len(tma_pending))):
                bars[name].arrive(1, phase)
            continue
        ev = cur[c]
        if ev[0] == "mma":
            mma_queue.append(ev[1])
        elif ev[0] == "tma":
            tma_pending.append(ev[1])
        elif ev[0] == "arrive":
            bars[ev[1]].arrive(ev[2], ev[3])
        nxt = next(agents[c], None)
        if nxt is None:
            del cur[c]
        else:
            cur[c] = nxt
    return steps
