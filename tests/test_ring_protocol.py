"""A model of the GEMM's shared-memory rings, run against every ring
configuration the kernel dispatches (parsed from its source).

The model keeps what matters for ordering: mbarriers with phase-parity
waits (a wait for parity P passes as soon as the barrier's current,
incomplete phase has the other parity), bulk copies that land after a
random delay (a few of them very late), tcgen05 commits that complete in
issue order, and the roles of the kernel:
  * the weight producer fills weight slot u % SW for unit u once the slot's
    previous fill has been consumed (wempty);
  * D dequant groups take the units in turn (group u % D).  Each waits for
    its weight fill (wfull), reads it, frees the slot (wempty), waits for a
    free A slot (xaempty), writes it and arrives on afull;
  * the X8 producer waits for a free X8 slot (xaempty) and issues its copy,
    which completes on the slot's own x8full (the producer's arrival plus
    the copy's bytes, nothing else);
  * the MMA waits on afull and x8full, consumes unit u, and its commit
    (after a delay) frees the X8/A slot (xaempty).
A second model (run_pair) covers two CTAs of a pair with an abort injected
at any step: CTA 1 forwards the landing of its X8 half to CTA 0 (x8peer),
and every producer drains only barriers its own copies complete, so every
issued copy has landed before the CTA exits.
Every consumer checks that what it reads is the unit it waited for, so a
wait that passes on another phase (aliasing) fails the test.  The model is
shown to catch the weight-slot race of an odd ring shared by two groups.
"""
import os
import random
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GEMM_SRC = os.path.join(ROOT, "w4a8_integer_gemm_b200", "csrc", "qoq_gemm.cu")


class Barrier:
    """An mbarrier: `count` arrivals plus any expected transaction bytes
    complete the current phase."""

    def __init__(self, count):
        self.count = count
        self.pending = count
        self.tx = 0
        self.completed = 0  # phases completed so far

    def passes(self, parity):
        # the current (incomplete) phase has parity completed % 2
        return (self.completed & 1) != parity

    def arrive(self, tx=0):
        self.pending -= 1
        self.tx += tx
        self._check()

    def complete_tx(self, tx):
        self.tx -= tx
        self._check()

    def _check(self):
        assert self.pending >= 0, "more arrivals than the phase expects"
        if self.pending == 0 and self.tx == 0:
            self.completed += 1
            self.pending = self.count


def run_rings(SW, SX, D, units, seed, steps=200000, ks=None, acc_bufs=2, epi=1, accempty_count=None):
    """ks: units per output tile (default: one tile); acc_bufs: TMEM
    accumulators; epi: epilogue groups, each draining every tile;
    accempty_count: the accempty arrival count (default: epi)."""
    rng = random.Random(seed)
    wfull = [Barrier(1) for _ in range(SW)]
    wempty = [Barrier(D and 1) for _ in range(SW)]
    afull = [Barrier(1) for _ in range(SX)]    # the dequant group
    x8full = [Barrier(1) for _ in range(SX)]   # the X8 producer and its copy's bytes
    xaempty = [Barrier(1) for _ in range(SX)]  # the MMA's commit
    wslot = [None] * SW                        # unit whose weights a slot holds
    xslot = [None] * SX                        # unit whose X8 tile an X8 slot holds
    # accumulators: the MMA waits for accempty before a tile and commits
    # accfull after its last unit; every epilogue group drains every tile
    ks = ks or units
    ntiles = (units + ks - 1) // ks
    accfull = [Barrier(1) for _ in range(acc_bufs)]
    accempty = [Barrier(accempty_count or epi) for _ in range(acc_bufs)]
    acc = [None] * acc_bufs                    # [tile, units accumulated, epilogue groups that read it]
    aslot = [None] * SX                        # unit whose dequantized weights an A slot holds
    inflight = []                              # [due time, sequence, action]
    clock = [0, 0]                             # now, sequence numbers
    last_commit = [0]

    def later(action, delay):
        clock[1] += 1
        inflight.append([clock[0] + delay, clock[1], action])

    def copy_delay():
        # most copies land soon; a few much later (a slow DRAM channel)
        return rng.randint(1, 30) if rng.random() < 0.9 else rng.randint(60, 400)

    def w_producer():
        for u in range(units):
            s, k = u % SW, u // SW
            while not wempty[s].passes((k & 1) ^ 1):
                yield
            wfull[s].arrive(tx=1)

            def land(s=s, u=u):
                wslot[s] = u
                wfull[s].complete_tx(1)
            later(land, copy_delay())
            yield

    def dequant(g):
        for u in range(g, units, D):
            s, k = u % SW, u // SW
            while not wfull[s].passes(k & 1):
                yield
            assert wslot[s] == u, f"dequant of unit {u} read weight slot {s} holding unit {wslot[s]}"
            yield
            wempty[s].arrive()
            a, j = u % SX, u // SX
            while not xaempty[a].passes((j & 1) ^ 1):
                yield
            assert aslot[a] is None, f"A slot {a} overwritten before the MMA read unit {aslot[a]}"
            aslot[a] = u
            yield
            afull[a].arrive()

    def x_producer():
        for u in range(units):
            a, j = u % SX, u // SX
            while not xaempty[a].passes((j & 1) ^ 1):
                yield
            assert xslot[a] is None, f"X8 slot {a} overwritten before the MMA read unit {xslot[a]}"
            x8full[a].arrive(tx=1)

            def land(a=a, u=u):
                xslot[a] = u
                x8full[a].complete_tx(1)
            later(land, copy_delay())
            yield

    def mma():
        for u in range(units):
            t = u // ks
            b, jt = t % acc_bufs, t // acc_bufs
            if u % ks == 0:
                while not accempty[b].passes((jt & 1) ^ 1):
                    yield
                assert acc[b] is None or acc[b][2] == epi, f"tile {t} overwrites accumulator {b} before it was drained"
                acc[b] = [t, 0, 0]
            a, j = u % SX, u // SX
            while not (afull[a].passes(j & 1) and x8full[a].passes(j & 1)):
                yield
            assert aslot[a] == u and xslot[a] == u, f"MMA of unit {u} read A {aslot[a]} and X8 {xslot[a]}"
            acc[b][1] += 1
            yield
            if u % ks == ks - 1 or u == units - 1:
                def acc_commit(b=b):
                    accfull[b].arrive()
                due = max(last_commit[0] + 1, clock[0] + rng.randint(1, 20))
                last_commit[0] = due
                later(acc_commit, due - clock[0])

            def commit(a=a):
                aslot[a] = None
                xslot[a] = None
                xaempty[a].arrive()
            # a commit completes after the MMAs it tracks, and after every
            # earlier commit
            due = max(last_commit[0] + 1, clock[0] + rng.randint(1, 20))
            last_commit[0] = due
            later(commit, due - clock[0])

    def epilogue(g):
        for t in range(ntiles):
            b, jt = t % acc_bufs, t // acc_bufs
            while not accfull[b].passes(jt & 1):
                yield
            expect = min(ks, units - t * ks)
            assert acc[b] is not None and acc[b][0] == t and acc[b][1] == expect, \
                f"epilogue group {g} read accumulator {b} as tile {t}: {acc[b]}"
            yield
            acc[b][2] += 1
            accempty[b].arrive()

    roles = [w_producer(), x_producer(), mma()] + [dequant(g) for g in range(D)] + [epilogue(g) for g in range(epi)]
    live = list(roles)
    for _ in range(steps):
        if not live and not inflight:
            return
        # either a role advances or time moves on, landing what is due
        if inflight and (not live or rng.random() < 0.5):
            clock[0] += 1
            done = sorted((f for f in inflight if f[0] <= clock[0]), key=lambda f: (f[0], f[1]))
            inflight[:] = [f for f in inflight if f[0] > clock[0]]
            for f in done:
                f[2]()
            continue
        r = rng.choice(live)
        try:
            next(r)
        except StopIteration:
            live.remove(r)
    raise AssertionError("the model did not finish (a wait that never passes)")


def dispatched_configs():
    """(BN, SW, SX, dequant groups) of every launch_cfg in the GEMM's
    dispatch table, both values of each `A_TMEM ? x : y`."""
    src = open(GEMM_SRC).read()
    body = src[src.index("cudaError_t dispatch(int BN, int KST, bool pair"):]
    body = body[:body.index("\n}\n")]
    out = set()
    for m in re.finditer(r"launch_cfg<([^>]*)>", body):
        args = [x.strip() for x in m.group(1).split(",")]
        bn = int(args[0])

        def pick(expr, tmem):
            t = re.match(r"A_TMEM \? (\d+) : (\d+)", expr)
            return int(t.group(1) if tmem else t.group(2)) if t else int(expr)
        for tmem in (True, False):
            out.add((bn, pick(args[2], tmem), pick(args[3], tmem), 2 if bn <= 64 else 1))
    return sorted(out)


def accumulator_configs():
    """(BN, KST, SX, A in TMEM, accumulator buffers, epilogue groups) of every
    dispatched configuration, with the kernel's rules for the last two (two
    accumulators where TMEM holds them beside the A ring; two epilogue
    groups for 256-token tiles)."""
    src = open(GEMM_SRC).read()
    assert "kAccBufs = (2 * BN + (A_TMEM ? SX * (int)kACols : 0) <= 512) ? 2 : 1;" in src, \
        "the kernel's accumulator-count rule changed: update this model"
    assert "epilogue_groups(int BN) { return BN == 256 ? 2 : 1; }" in src
    body = src[src.index("cudaError_t dispatch(int BN, int KST, bool pair"):]
    body = body[:body.index("\n}\n")]
    out = set()
    for m in re.finditer(r"launch_cfg<([^>]*)>", body):
        args = [x.strip() for x in m.group(1).split(",")]
        bn, kst = int(args[0]), int(args[1])
        flag = args[4]
        for tmem in ((True, False) if flag == "A_TMEM" else (flag == "true",)):
            t = re.match(r"A_TMEM \? (\d+) : (\d+)", args[3])
            sx = int(t.group(1) if tmem else t.group(2)) if t else int(args[3])
            bufs = 2 if 2 * bn + (sx * (kst // 4) if tmem else 0) <= 512 else 1
            out.add((bn, kst, sx, tmem, bufs, 2 if bn == 256 else 1))
    return sorted(out)


@pytest.mark.parametrize("cfg", accumulator_configs(), ids=lambda c: "BN%d_KST%d_SX%d_tmem%d_acc%d_epi%d" % c)
def test_accumulator_handoff(cfg):
    bn, kst, SX, tmem, bufs, epi = cfg
    D = 2 if bn <= 64 else 1
    for seed in range(20):
        for ks in (1, 3, 4):
            run_rings(2 * SX, SX, D, units=4 * ks + 3, seed=seed, ks=ks, acc_bufs=bufs, epi=epi)


def test_the_model_catches_an_accumulator_released_by_one_of_two_groups():
    # accempty expecting one arrival where two epilogue groups drain each tile:
    # a tile overwrites an undrained accumulator, or the ring deadlocks
    with pytest.raises(AssertionError, match="accumulator|did not finish"):
        for seed in range(200):
            run_rings(4, 2, 1, units=20, seed=seed, ks=2, acc_bufs=1, epi=2, accempty_count=1)


def test_dispatch_table_parsed():
    cfgs = dispatched_configs()
    assert len(cfgs) >= 12
    assert (64, 8, 5, 2) in cfgs and (16, 10, 7, 2) in cfgs and (256, 5, 4, 1) in cfgs


@pytest.mark.parametrize("cfg", dispatched_configs(), ids=lambda c: "BN%d_SW%d_SX%d_D%d" % c)
def test_rings_of_every_dispatched_configuration(cfg):
    bn, SW, SX, D = cfg
    for seed in range(30):
        run_rings(SW, SX, D, units=3 * SW + 5, seed=seed)


def test_the_model_catches_a_weight_slot_shared_by_two_groups():
    # the depths the 64-token decode configuration had: an odd weight ring
    # (7) shared by two dequant groups with an X8/A ring of 6
    with pytest.raises(AssertionError, match="read weight slot"):
        for seed in range(400):
            run_rings(7, 6, 2, units=40, seed=seed)


# ------------------------------------------------------------------------
# CTA pairs and aborts
# ------------------------------------------------------------------------
def run_pair(SW, SX, units, seed, abort_at=None, abort_cta=0, pair=True, own_x8_barrier=True,
             drain_ticks=5000, peer_drain=True, steps=400000):
    """Two CTAs (or one, pair=False) of the kernel's rings with an abort.

    Each CTA has a weight producer, one dequant group and an X8 producer;
    CTA 0 issues the MMAs and multicasts each commit to both CTAs' xaempty,
    and both CTAs' dequant groups arrive on CTA 0's afull.  With
    own_x8_barrier (the kernel's design): CTA 0's X8 copies complete on its
    own x8full; CTA 1's producer arms CTA 0's x8peer itself (a remote
    arrival expecting its half's bytes) and its copy completes there; the
    MMA waits on afull, x8full and x8peer.  Without it (the earlier
    design), the producer's arrival and the copy's bytes counted on afull,
    which also needs the dequant arrivals.

    At step abort_at, CTA abort_cta raises its abort flag (as a timed-out
    wait does).  A role whose wait is not yet satisfied leaves when its
    CTA's flag is up; a wait that stays unsatisfied for 2000 ticks raises
    the flag (the kernel's per-wait budget).  End of the kernel, as in the
    source: the CTA's roles meet (block barrier); if its flag is up, its
    producers wait for their own copies' barrier phases (the earlier
    design: for at most drain_ticks, its grace period); a pair then meets
    at a cluster barrier (CTA 1 has stated how many stages it issued),
    CTA 0 (if either CTA aborted) waits for the latest x8peer phase of every slot CTA 1
    used (each completes exactly when its copy lands; peer_drain=False
    skips this), and the pair meets again before exiting.  The model
    checks that no copy lands in a CTA after it exited."""
    rng = random.Random(seed)
    ncta = 2 if pair else 1
    clock = [0, 0]
    inflight = []
    last_commit = [0]
    abort = [False] * ncta
    nroles = [0] * ncta
    done_roles = [0] * ncta      # roles past the block barrier
    drained = [0] * ncta         # roles past their own drains
    peer_drained = [False]
    exited = [False] * ncta

    def later(action, delay):
        clock[1] += 1
        inflight.append([clock[0] + delay, clock[1], action])

    def copy_delay():
        return rng.randint(1, 30) if rng.random() < 0.9 else rng.randint(60, 400)

    wfull = [[Barrier(1) for _ in range(SW)] for _ in range(ncta)]
    wempty = [[Barrier(1) for _ in range(SW)] for _ in range(ncta)]
    x8full = [Barrier(1) for _ in range(SX)]          # CTA 0's own X8 copies
    x8peer = [Barrier(1) for _ in range(SX)]          # in CTA 0: CTA 1's half (armed by CTA 1)
    n_peer = [0]                                      # stages CTA 1 issued
    if own_x8_barrier:
        afull = [Barrier(ncta) for _ in range(SX)]            # both CTAs' dequant groups
    else:
        afull = [Barrier(ncta + 1) for _ in range(SX)]        # + CTA 0's producer (both halves' bytes)
    xaempty = [[Barrier(1) for _ in range(SX)] for _ in range(ncta)]
    wslot = [[None] * SW for _ in range(ncta)]
    xslot = [[None] * SX for _ in range(ncta)]
    aslot = [[None] * SX for _ in range(ncta)]
    drains = [[] for _ in range(ncta)]   # (barrier, parity, bounded, owner)

    def landing(c, fn):
        def act():
            assert not exited[c], f"a copy landed in CTA {c} after it exited"
            fn()
        return act

    def waiting(c, cond, budget=2000):
        t0 = clock[0]
        while not cond():
            if abort[c]:
                return
            if clock[0] - t0 > budget:
                abort[c] = True
                return
            yield
        return True

    def drain(bar, par, bounded):
        waited = 0
        while not bar.passes(par):
            if bounded and waited >= drain_ticks:
                return
            waited += 1
            yield

    def role(c, gen, owner=None):
        nroles[c] += 1

        def run():
            yield from gen
            done_roles[c] += 1
            while done_roles[c] < nroles[c]:                   # block barrier
                yield
            if abort[c] and owner is not None:
                for bar, par, bounded, o in drains[c]:
                    if o == owner:
                        yield from drain(bar, par, bounded)
            drained[c] += 1
            if pair:
                while sum(drained) < sum(nroles):              # cluster barrier 1
                    yield
                if c == 0 and owner == "x8" and any(abort) and peer_drain:
                    n1 = n_peer[0]
                    for a in range(min(SX, n1)):
                        j = a + (n1 - 1 - a) // SX * SX       # CTA 1's last stage in slot a
                        yield from drain(x8peer[a], (j // SX) & 1, False)
                    peer_drained[0] = True
                elif c == 0 and owner == "x8":
                    peer_drained[0] = True
                while not peer_drained[0]:                     # cluster barrier 2
                    yield
            else:
                while drained[c] < nroles[c]:
                    yield
            exited[c] = True
        return run()

    def w_producer(c):
        issued = {}
        for u in range(units):
            s, k = u % SW, u // SW
            ok = yield from waiting(c, lambda s=s, k=k: wempty[c][s].passes((k & 1) ^ 1))
            if not ok:
                break
            wfull[c][s].arrive(tx=1)
            issued[s] = k & 1

            def land(s=s, u=u):
                wslot[c][s] = u
                wfull[c][s].complete_tx(1)
            later(landing(c, land), copy_delay())
            yield
        drains[c].extend((wfull[c][s], par, False, "w") for s, par in issued.items())

    def dequant(c):
        for u in range(units):
            s, k = u % SW, u // SW
            ok = yield from waiting(c, lambda s=s, k=k: wfull[c][s].passes(k & 1))
            if not ok:
                return
            assert wslot[c][s] == u
            yield
            wempty[c][s].arrive()
            a, j = u % SX, u // SX
            ok = yield from waiting(c, lambda a=a, j=j: xaempty[c][a].passes((j & 1) ^ 1))
            if not ok:
                return
            aslot[c][a] = u
            yield
            afull[a].arrive()

    def x_producer(c):
        issued = {}
        for u in range(units):
            a, j = u % SX, u // SX
            ok = yield from waiting(c, lambda a=a, j=j: xaempty[c][a].passes((j & 1) ^ 1))
            if not ok:
                break
            if not own_x8_barrier:
                bar = afull[a]
                if c == 0:
                    bar.arrive(tx=ncta)            # both halves' bytes
                issued[a] = (bar, j & 1, True)
            elif c == 0:
                bar = x8full[a]
                bar.arrive(tx=1)
                issued[a] = (bar, j & 1, False)
            else:
                # CTA 1: arms CTA 0's x8peer itself; its bytes complete there
                bar = x8peer[a]
                bar.arrive(tx=1)
                n_peer[0] += 1

            def land(a=a, u=u, bar=bar):
                xslot[c][a] = u
                bar.complete_tx(1)
            later(landing(c, land), copy_delay())
            yield
        drains[c].extend((bar, par, bounded, "x8") for a, (bar, par, bounded) in issued.items())

    def mma():
        for u in range(units):
            a, j = u % SX, u // SX

            def ready(a=a, j=j):
                if not afull[a].passes(j & 1):
                    return False
                if own_x8_barrier:
                    if not x8full[a].passes(j & 1):
                        return False
                    if pair and not x8peer[a].passes(j & 1):
                        return False
                return True
            ok = yield from waiting(0, ready)
            if not ok:
                return
            for c in range(ncta):
                assert aslot[c][a] == u and xslot[c][a] == u, f"MMA of unit {u}: CTA {c} A {aslot[c][a]} X8 {xslot[c][a]}"
            yield

            def commit(a=a):
                for c in range(ncta):
                    aslot[c][a] = None
                    xslot[c][a] = None
                    xaempty[c][a].arrive()
            due = max(last_commit[0] + 1, clock[0] + rng.randint(1, 20))
            last_commit[0] = due
            later(commit, due - clock[0])

    live = []
    for c in range(ncta):
        live += [role(c, w_producer(c), "w"), role(c, dequant(c)), role(c, x_producer(c), "x8")]
    live.append(role(0, mma()))
    step = 0
    while live or inflight:
        step += 1
        if step > steps:
            raise AssertionError("the model did not finish (a wait that never passes)")
        if abort_at is not None and step == abort_at:
            for c in (range(ncta) if abort_cta == "both" else (abort_cta,)):
                abort[c] = True
        # time moves on (landing what is due) about every other step, also
        # while nothing is in flight (the per-wait budgets run on it)
        if not live or rng.random() < 0.5:
            clock[0] += 1
            done = sorted((f for f in inflight if f[0] <= clock[0]), key=lambda f: (f[0], f[1]))
            inflight[:] = [f for f in inflight if f[0] > clock[0]]
            for f in done:
                f[2]()
            continue
        r = rng.choice(live)
        try:
            next(r)
        except StopIteration:
            live.remove(r)
    return abort


@pytest.mark.parametrize("pair", [False, True], ids=["single", "pair"])
def test_pair_rings_without_abort(pair):
    for seed in range(30):
        run_pair(4, 4, units=23, seed=seed, pair=pair)


@pytest.mark.parametrize("pair", [False, True], ids=["single", "pair"])
@pytest.mark.parametrize("abort_cta", [0, 1, "both"])
def test_abort_at_every_step_lets_every_copy_land(pair, abort_cta):
    """An abort at any step, in either CTA or both: every issued copy lands
    before its CTA exits, and no role waits forever."""
    if not pair and abort_cta != 0:
        pytest.skip("one CTA")
    for seed in range(4):
        for at in range(1, 400, 4):
            run_pair(4, 4, units=18, seed=seed, abort_at=at, abort_cta=abort_cta, pair=pair)


def test_the_model_catches_the_earlier_x8_drain():
    """With X8 bytes counted on afull (which also needs the dequant
    arrivals) and a bounded grace period, some abort leaves a copy landing
    after the CTA exited."""
    with pytest.raises(AssertionError, match="landed in CTA"):
        for seed in range(60):
            for at in range(1, 300, 2):
                run_pair(4, 4, units=18, seed=seed, abort_at=at, pair=False, own_x8_barrier=False,
                         drain_ticks=5)


def test_the_model_catches_a_pair_leaving_before_the_peer_drain():
    """Without CTA 0's wait for CTA 1's x8peer phases, CTA 1 can exit while
    its last copy is still landing."""
    with pytest.raises(AssertionError, match="landed in CTA 1"):
        for seed in range(80):
            for at in range(1, 300, 3):
                run_pair(4, 4, units=18, seed=seed, abort_at=at, abort_cta="both", pair=True, peer_drain=False)
