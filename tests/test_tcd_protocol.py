"""A discrete model of the decode tensor-core GEMM's barrier protocol (path 6,
`gemm_tcd.cu`), checked on the CPU.

The kernel's roles hand data to each other only through mbarriers whose waits name
a phase by its parity.  A parity names a phase only to a waiter at most one phase
away, so the kernel keeps one rule: every waiter of a barrier waits on each of its
phases in order.  This model runs the roles of one CTA as Python generators, with
random delays, copies that land and MMAs that complete at random later times (in
issue order per issuing thread, in any order across threads).  It has the same ring
sizes, chunk alignment and walk over (row tile, K range) units as the kernel.  For
every unit list of a grid of tiles, splits and CTAs it checks that:
  - every role finishes (no deadlock);
  - every read sees the bytes of the k-block it expects: raw codes when widened,
    operand and tokens when an MMA executes, an accumulator when drained.
A negative control breaks the rule (a widening group that skips the weight chunks
holding none of its k-blocks) and must be caught.
"""
import random

import pytest


class Bar:
    """An mbarrier: an arrival count per phase, a transaction byte count, phases completed."""

    def __init__(self, name, count):
        self.name, self.count, self.pending, self.tx, self.done_phases = name, count, count, 0, 0

    def arrive(self, tx=0):
        self.tx += tx
        self.pending -= 1
        assert self.pending >= 0, f"{self.name}: more arrivals than its count"
        self._check()

    def complete_tx(self, n):
        self.tx -= n
        assert self.tx >= 0, f"{self.name}: more bytes than expected"
        self._check()

    def _check(self):
        if self.pending == 0 and self.tx == 0:
            self.done_phases += 1
            self.pending = self.count

    def passed(self, parity):
        # try_wait.parity: true when the phase of this parity is the last one completed
        return (self.done_phases & 1) != parity


# ring sizes per token tile NT, as in gemm_tcd.cu's Cfg<NT>:
# (A stages, B stages, B chunk, R slots, widening groups, accumulators, epilogue warps)
CFG = {16: (4, 12, 4, 16, 4, 8, 4), 32: (4, 12, 4, 12, 4, 8, 4),
       64: (4, 6, 2, 12, 2, 8, 8), 128: (4, 4, 2, 8, 2, 4, 8)}
KCR = 4       # R slots per weight chunk
GW = 2        # warps per widening group


def units_of(kblocks, S, t8, t4, grid, cta):
    """The (8-bit?, kb0, kb1) units CTA `cta` walks: u = cta, cta + grid, ..."""
    per = -(-kblocks // S)
    S = -(-kblocks // per)
    return [(u // S < t8, (u % S) * per, min(kblocks, (u % S) * per + per))
            for u in range(cta, (t8 + t4) * S, grid)]


def run(units, NT, gpk, seed, skip_foreign_chunks=False):
    kA, kB, kCB, kR, G, kSlots, E = CFG[NT]
    rng = random.Random(seed)
    nch = kB // kCB
    r_full = [Bar(f"r_full{i}", 1) for i in range(kR)]
    r_rel = [Bar(f"r_rel{i}", G * GW) for i in range(kR // KCR)]
    b_full = [Bar(f"b_full{i}", 1) for i in range(kB)]
    b_empty = [Bar(f"b_empty{i}", 2) for i in range(nch)]
    ready = [Bar(f"ready{i}", GW) for i in range(kA)]
    a_empty = [Bar(f"a_empty{i}", gpk) for i in range(kA)]
    acc_full = [Bar(f"acc_full{i}", 1) for i in range(kSlots)]
    acc_empty = [Bar(f"acc_empty{i}", E) for i in range(kSlots)]
    landing = []                       # copies in flight
    tensor = [[], []]                  # each issuer's MMAs and commits, completed in order
    r_tag, b_tag, a_tag, acc_tag = [None] * kR, [None] * kB, [None] * kA, [None] * kSlots
    kb_of = [(u, kb) for u, (_, k0, k1) in enumerate(units) for kb in range(k0, k1)]

    def weights():                     # warp 0: chunks of KCR slots aligned to the ring
        ir, runs = 0, []

        def flush(end):
            base = (end - 1) & ~(KCR - 1)
            yield r_rel[(base % kR) // KCR], ((base // kR) & 1) ^ 1
            r_full[base % kR].arrive(sum(n for _, _, n in runs))
            for slot, tags, n in list(runs):
                def land(slot=slot, tags=tags, n=n, base=base):
                    for j, t in enumerate(tags):
                        r_tag[(slot + j) % kR] = t
                    r_full[base % kR].complete_tx(n)
                landing.append(land)
            runs.clear()
        for u, (eight, kb0, kb1) in enumerate(units):
            w = 2 if eight else 1
            ns, o = (kb1 - kb0) * w, 0
            while o < ns:
                take = min(ns - o, KCR - ir % KCR)
                assert ir % kR + take <= kR, "a chunk wraps the R ring"
                runs.append((ir, [(u, kb0 + (o + j) // w, (o + j) % w) for j in range(take)], take))
                ir, o = ir + take, o + take
                if ir % KCR == 0:
                    yield from flush(ir)
        if ir % KCR:
            yield from flush(ir)

    def tokens():                      # warp 3: chunks of kCB k-blocks aligned to the ring
        ia = 0

        def flush(end):
            base = (end - 1) & ~(kCB - 1)
            ci = base // kCB
            yield b_empty[ci % nch], ((ci // nch) & 1) ^ 1
            b_full[base % kB].arrive(end - base)
            for st in range(base, end):
                def land(st=st, base=base):
                    b_tag[st % kB] = kb_of[st]
                    b_full[base % kB].complete_tx(1)
                landing.append(land)
        for _, (_, kb0, kb1) in enumerate(units):
            kb = kb0
            while kb < kb1:
                take = min(kb1 - kb, kCB - ia % kCB)
                assert ia % kB + take <= kB, "a chunk wraps the B ring"
                ia, kb = ia + take, kb + take
                if ia % kCB == 0:
                    yield from flush(ia)
        if ia % kCB:
            yield from flush(ia)

    def issuer(mine):                  # warps 1-2: every second group
        ia = gc = 0
        seen, any_mma = -1, False
        q = tensor[mine]
        for u, (_, kb0, kb1) in enumerate(units):
            last_unit = u == len(units) - 1
            for kb in range(kb0, kb1):
                sa, sb = ia % kA, ia % kB
                if gpk == 2 or (gc & 1) == mine:
                    hb = ia & ~(kCB - 1)
                    if hb != seen:
                        yield b_full[hb % kB], (hb // kB) & 1
                        seen = hb
                    yield ready[sa], (ia // kA) & 1
                    for _ in range(gpk):
                        if (gc & 1) != mine:
                            gc += 1
                            continue
                        b = gc % kSlots
                        yield acc_empty[b], (gc // kSlots) & 1

                        def execute(sa=sa, sb=sb, want=(u, kb), b=b, gc=gc):
                            assert a_tag[sa] == want, ("operand", a_tag[sa], want)
                            assert b_tag[sb] == want, ("tokens", b_tag[sb], want)
                            acc_tag[b] = gc
                        q.append(execute)
                        q.append(acc_full[b].arrive)
                        q.append(a_empty[sa].arrive)
                        any_mma = True
                        gc += 1
                else:
                    gc += 1
                if (ia + 1) % kCB == 0 or (last_unit and kb + 1 == kb1):
                    # only the CTA's last chunk can hold no k-block of this issuer; no copy
                    # waits on that chunk's release, so there is nothing to arrive for
                    if any_mma:
                        q.append(b_empty[(ia // kCB) % nch].arrive)
                    any_mma = False
                ia += 1

    def widening(g):                   # warps 4-: group g widens k-blocks ia % G == g
        ir = ia = 0
        entered, released = -KCR, 0
        for u, (eight, kb0, kb1) in enumerate(units):
            w = 2 if eight else 1
            for kb in range(kb0, kb1):
                mine = ia % G == g
                while entered + KCR <= ir + w - 1:
                    entered += KCR
                    own = entered <= ir + w - 1 and entered + KCR > ir
                    if not (skip_foreign_chunks and not (mine and own)):
                        yield r_full[entered % kR], (entered // kR) & 1
                if mine:
                    sa = ia % kA
                    yield a_empty[sa], ((ia // kA) & 1) ^ 1
                    assert r_tag[ir % kR] == (u, kb, 0), ("raw", r_tag[ir % kR], (u, kb))
                    if w == 2:
                        assert r_tag[(ir + 1) % kR] == (u, kb, 1), ("raw", r_tag[(ir + 1) % kR], (u, kb))
                    a_tag[sa] = (u, kb)
                    for _ in range(GW):
                        ready[sa].arrive()
                while released + KCR <= ir + w:
                    for _ in range(GW):
                        r_rel[(released % kR) // KCR].arrive()
                    released += KCR
                ia, ir = ia + 1, ir + w
        while released <= entered:
            for _ in range(GW):
                r_rel[(released % kR) // KCR].arrive()
            released += KCR

    def epilogue():                    # the epilogue warps, in step
        for bar in acc_empty:
            for _ in range(E):
                bar.arrive()
        gc = 0
        for _, (_, kb0, kb1) in enumerate(units):
            for _ in range(kb0 * gpk, kb1 * gpk):
                b = gc % kSlots
                yield acc_full[b], (gc // kSlots) & 1
                assert acc_tag[b] == gc, ("accumulator", acc_tag[b], gc)
                for _ in range(E):
                    acc_empty[b].arrive()
                gc += 1

    roles = [weights(), tokens(), issuer(0), issuer(1), epilogue()] + [widening(g) for g in range(G)]
    waiting = [None] * len(roles)
    alive = list(range(len(roles)))
    while alive or landing or tensor[0] or tensor[1]:
        moved = False
        for i in rng.sample(alive, len(alive)):
            if waiting[i] is not None and not waiting[i][0].passed(waiting[i][1]):
                continue
            if rng.random() < 0.3:                      # a role late this round
                continue
            try:
                waiting[i] = next(roles[i])
            except StopIteration:
                alive.remove(i)
                waiting[i] = None
            moved = True
        if landing and rng.random() < 0.3:
            landing.pop(rng.randrange(len(landing)))()
            moved = True
        for q in tensor:
            if q and rng.random() < 0.3:
                q.pop(0)()
                moved = True
        if not moved:
            if landing:
                landing.pop(0)()
                continue
            if tensor[0] or tensor[1]:
                (tensor[0] or tensor[1]).pop(0)()
                continue
            if any(waiting[i] is None or waiting[i][0].passed(waiting[i][1]) for i in alive):
                continue
            return "deadlock: " + ", ".join(f"{waiting[i][0].name}@{waiting[i][1]}" for i in alive)
    return "ok"


def unit_lists():
    for kblocks in (1, 3, 4, 7, 10, 33):
        for S in (1, 2, 3, 7):
            for t8, t4 in ((1, 3), (0, 2), (3, 5)):
                for grid in (1, 3):
                    un = units_of(kblocks, S, t8, t4, grid, 0)
                    if un:
                        yield un


@pytest.mark.parametrize("NT", [16, 32, 64, 128])
@pytest.mark.parametrize("gpk", [1, 2])
def test_protocol_finishes_and_every_read_sees_its_kblock(NT, gpk):
    for i, un in enumerate(unit_lists()):
        for seed in range(2):
            try:
                r = run(un, NT, gpk, seed=1000 * i + seed)
            except AssertionError as e:
                r = f"wrong data: {e}"
            assert r == "ok", (NT, gpk, un, r)


def test_model_catches_a_group_that_skips_chunks_of_other_groups():
    # the rule broken: a widening group waits only on the weight chunks that hold its own
    # k-blocks, so it may wait on a chunk barrier two phases away from its last wait
    bad = 0
    for i, un in enumerate(unit_lists()):
        for seed in range(3):
            try:
                r = run(un, 16, 1, seed=77 * i + seed, skip_foreign_chunks=True)
            except AssertionError as e:
                r = f"wrong data: {e}"
            bad += r != "ok"
    assert bad > 0
