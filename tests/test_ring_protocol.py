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
  * the X8 producer waits for a free X8 slot (xaempty) and issues its copy
    (afull completes on its bytes);
  * the MMA waits on afull, consumes unit u, and its commit (after a delay)
    frees the X8/A slot (xaempty).
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
    afull = [Barrier(2) for _ in range(SX)]    # the dequant group + the X8 producer (and its bytes)
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
            afull[a].arrive(tx=1)

            def land(a=a, u=u):
                xslot[a] = u
                afull[a].complete_tx(1)
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
            while not afull[a].passes(j & 1):
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
