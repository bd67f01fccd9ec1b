"""A discrete model of the prefill tensor-core GEMM's barrier protocol on CTA pairs
(path 5, `gemm_tc3.cu`), checked on the CPU.

The pair shares its barriers across the cluster:
  - each CTA's copy warps wait on their own CTA's "empty" barrier;
  - the widening warps of both CTAs arrive on the even CTA's "ready" barrier;
  - the even CTA's two MMA issuers commit to the "empty" and "accumulator full" barriers
    of both CTAs;
  - the epilogue warps of both CTAs release an accumulator on the even CTA's barrier.

Every parity wait must name a phase at most one away.  The model runs the roles of both
CTAs as Python generators: random delays, copies that land and MMAs that complete at
random later times (in issue order per issuing thread).  It has the kernel's stage and
accumulator counts and its walk over (row-tile pair, token tile) units, a CTA past the
last row tile included.  For every unit walk it checks that every role finishes, that
every MMA executes on the k-block's operands and tokens in both CTAs, and that every
drain reads the group it expects.
"""
import random

import pytest

from test_tcd_protocol import Bar

K_STAGES, K_SLOTS = 5, 2          # gemm_tc3.cu: kStages, kSlots
W, E = 4, 8                       # widening and epilogue warps per CTA


def run(units, nkb, gpk, seed, early_release=False):
    """units: per unit of this cluster, the rows flag of each CTA ((rows0, rows1), unit id)."""
    rng = random.Random(seed)
    full_w = [[Bar(f"full_w{r}.{s}", 1) for s in range(K_STAGES)] for r in range(2)]
    full_t = [[Bar(f"full_t{r}.{s}", 1) for s in range(K_STAGES)] for r in range(2)]
    empty = [[Bar(f"empty{r}.{s}", gpk) for s in range(K_STAGES)] for r in range(2)]
    acc_full = [[Bar(f"acc_full{r}.{b}", 1) for b in range(K_SLOTS)] for r in range(2)]
    ready = [Bar(f"ready{s}", 2 * W) for s in range(K_STAGES)]          # even CTA
    acc_empty = [Bar(f"acc_empty{b}", 2 * E) for b in range(K_SLOTS)]  # even CTA
    landing, tensor = [], [[], []]
    a_tag = [[None] * K_STAGES for _ in range(2)]
    b_tag = [[None] * K_STAGES for _ in range(2)]
    acc_tag = [[None] * K_SLOTS for _ in range(2)]

    def weights(r):
        it = 0
        for (rows, u) in units:
            for kb in range(nkb):
                s, ph = it % K_STAGES, (it // K_STAGES) & 1
                yield empty[r][s], ph ^ 1
                if rows[r]:
                    full_w[r][s].arrive(1)

                    def land(s=s, t=(u, kb), r=r):
                        a_tag[r][s] = ("raw", t)
                        full_w[r][s].complete_tx(1)
                    landing.append(land)
                else:
                    full_w[r][s].arrive(0)                # a CTA without rows: nothing to copy
                it += 1

    def tokens(r):
        it = 0
        for (_, u) in units:
            for kb in range(nkb):
                s, ph = it % K_STAGES, (it // K_STAGES) & 1
                yield empty[r][s], ph ^ 1
                full_t[r][s].arrive(1)

                def land(s=s, t=(u, kb), r=r):
                    b_tag[r][s] = t
                    full_t[r][s].complete_tx(1)
                landing.append(land)
                it += 1

    def widening(r):                   # the W warps of CTA r, in step
        it = 0
        for (rows, u) in units:
            for kb in range(nkb):
                s, ph = it % K_STAGES, (it // K_STAGES) & 1
                yield full_w[r][s], ph
                yield full_t[r][s], ph
                if rows[r]:
                    assert a_tag[r][s] == ("raw", (u, kb)), ("raw", r, a_tag[r][s], (u, kb))
                    a_tag[r][s] = (u, kb)                # widened in place
                for _ in range(W):
                    ready[s].arrive()
                it += 1

    def issuer(mine):                  # the even CTA's MMA threads: accumulator `mine`
        it = gc = 0
        q = tensor[mine]
        for (rows, u) in units:
            for kb in range(nkb):
                s, ph = it % K_STAGES, (it // K_STAGES) & 1
                if gpk == 1 and (gc & 1) != mine:
                    gc += 1
                    it += 1
                    continue
                yield ready[s], ph
                for _ in range(gpk):
                    b = gc % K_SLOTS
                    if b != mine:
                        gc += 1
                        continue
                    yield acc_empty[b], (gc // K_SLOTS) & 1

                    def execute(s=s, want=(u, kb), rows=rows, b=b, gc=gc):
                        for r in range(2):
                            if rows[r]:
                                assert a_tag[r][s] == want, ("operand", r, a_tag[r][s], want)
                            assert b_tag[r][s] == want, ("tokens", r, b_tag[r][s], want)
                            acc_tag[r][b] = gc
                    q.append(execute)
                    for r in range(2):
                        q.append(acc_full[r][b].arrive)
                    for r in range(2):
                        q.append(empty[r][s].arrive)
                    gc += 1
                it += 1

    def epilogue(r):                   # the E warps of CTA r, in step
        for b in range(K_SLOTS):
            for _ in range(E):
                acc_empty[b].arrive()
        gc = 0
        for _ in units:
            for _ in range(nkb * gpk):
                b = gc % K_SLOTS
                yield acc_full[r][b], (gc // K_SLOTS) & 1
                if early_release:                # broken on purpose: release, then drain later
                    for _ in range(E):
                        acc_empty[b].arrive()
                    yield acc_full[r][b], (gc // K_SLOTS) & 1
                assert acc_tag[r][b] == gc, ("accumulator", r, acc_tag[r][b], gc)
                if not early_release:
                    for _ in range(E):
                        acc_empty[b].arrive()
                gc += 1

    roles = [weights(0), weights(1), tokens(0), tokens(1), widening(0), widening(1),
             issuer(0), issuer(1), epilogue(0), epilogue(1)]
    waiting = [None] * len(roles)
    alive = list(range(len(roles)))
    while alive or landing or any(tensor):
        moved = False
        for i in rng.sample(alive, len(alive)):
            if waiting[i] is not None and not waiting[i][0].passed(waiting[i][1]):
                continue
            if rng.random() < 0.3:
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
            busy = [q for q in tensor if q]
            if busy:
                busy[0].pop(0)()
                continue
            if any(waiting[i] is None or waiting[i][0].passed(waiting[i][1]) for i in alive):
                continue
            return "deadlock: " + ", ".join(f"{waiting[i][0].name}@{waiting[i][1]}" for i in alive)
    return "ok"


def walk(tiles, n_tt, n_clusters, cid):
    """The units cluster `cid` walks: u = cid, cid + n_clusters, ...; CTA r of the pair has
    row tile 2 (u / n_tt) + r, which may lie past the last tile."""
    pairs = (tiles + 1) // 2
    out = []
    for u in range(cid, pairs * n_tt, n_clusters):
        rt0 = 2 * (u // n_tt)
        out.append(((rt0 < tiles, rt0 + 1 < tiles), u))
    return out


@pytest.mark.parametrize("gpk", [1, 2])
def test_pair_protocol_finishes_and_every_read_sees_its_kblock(gpk):
    n = 0
    for tiles in (1, 2, 3, 5):
        for n_tt in (1, 2, 3):
            for n_clusters in (1, 2, 3):
                for nkb in (1, 2, 3, 5, 7):
                    units = walk(tiles, n_tt, n_clusters, 0)
                    if not units:
                        continue
                    for seed in range(2):
                        n += 1
                        try:
                            r = run(units, nkb, gpk, seed=31 * n + seed)
                        except AssertionError as e:
                            r = f"wrong data: {e}"
                        assert r == "ok", (tiles, n_tt, n_clusters, nkb, gpk, r)
    assert n > 100


def test_model_catches_an_accumulator_released_before_its_drain():
    caught = 0
    for n_tt in (2, 3):
        for nkb in (3, 5, 7):
            units = walk(5, n_tt, 1, 0)
            for seed in range(4):
                try:
                    r = run(units, nkb, 1, seed=seed, early_release=True)
                except AssertionError as e:
                    r = f"wrong data: {e}"
                caught += r != "ok"
    assert caught > 0
