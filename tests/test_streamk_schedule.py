"""The GEMM's stream-K schedule, checked on the CPU with the kernel's own
range arithmetic (the two device functions are parsed from the source):
the CTAs' unit ranges partition the work, and the split-tile roles the
epilogue derives from them are the ones its waits rely on -- a split tile is
finished by its first contributor, for which it is the last tile of its
range; every other contributor publishes it as the first tile of its range;
no CTA publishes or finishes twice."""
import os
import random
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GEMM_SRC = os.path.join(ROOT, "w4a8_integer_gemm_b200", "csrc", "qoq_gemm.cu")


def _device_fn(name):
    """The return expression of a one-line `int name(int a, int P, int T)`
    device function, as a Python function on non-negative integers."""
    src = open(GEMM_SRC).read()
    m = re.search(r"int %s\(int (\w+), int P, int T\)\s*\{\s*return (.*?);\s*\}" % name, src, re.S)
    assert m, name
    var, expr = m.group(1), m.group(2)
    expr = expr.replace("(long long)", "").replace("(int)", "").replace("/", "//")
    return eval("lambda %s, P, T: %s" % (var, expr))


cta_of = _device_fn("cta_of")
range_begin = _device_fn("range_begin")


def roles(P, tiles, ks):
    """Per CTA: the (tile, ks0, ks1, role) it works on, with the role the
    epilogue gives it (whole / finisher / publisher)."""
    T = tiles * ks
    out = []
    for c in range(P):
        b, e = range_begin(c, P, T), range_begin(c + 1, P, T)
        mine = []
        i = b
        while i < e:
            t = i // ks
            ks0 = i - t * ks
            ks1 = min(ks, e - t * ks)
            partial = not (ks0 == 0 and ks1 == ks)
            c_lo = cta_of(t * ks, P, T) if partial else c
            role = "whole" if not partial else ("finisher" if c_lo == c else "publisher")
            mine.append((t, ks0, ks1, role))
            i = t * ks + ks1
        out.append(mine)
    return out


def check(P, tiles, ks):
    T = tiles * ks
    # the ranges partition [0, T), and cta_of inverts them
    assert range_begin(0, P, T) == 0 and range_begin(P, P, T) == T
    for c in range(P):
        b, e = range_begin(c, P, T), range_begin(c + 1, P, T)
        assert b <= e
        for i in (b, e - 1) if e > b else ():
            assert cta_of(i, P, T) == c, (P, tiles, ks, c, i)
    rs = roles(P, tiles, ks)
    finished = {}
    published = {}
    for c, mine in enumerate(rs):
        assert sum(1 for r in mine if r[3] == "finisher") <= 1
        assert sum(1 for r in mine if r[3] == "publisher") <= 1
        for j, (t, ks0, ks1, role) in enumerate(mine):
            if role == "finisher":
                assert j == len(mine) - 1 and ks0 == 0 and ks1 < ks   # its last tile, from the start
                finished[t] = c
            elif role == "publisher":
                assert j == 0 and ks0 > 0                             # its first tile, mid-tile
                published.setdefault(t, []).append(c)
    for t in range(tiles):
        c_lo, c_hi = cta_of(t * ks, P, T), cta_of(t * ks + ks - 1, P, T)
        if c_lo == c_hi:
            assert t not in finished and t not in published
        else:
            # the finisher waits for exactly the CTAs (c_lo, c_hi], each publishing once
            assert finished[t] == c_lo
            assert sorted(published[t]) == list(range(c_lo + 1, c_hi + 1))


def test_schedule_properties_over_many_grids():
    rng = random.Random(7)
    cases = [(148, 112, 16), (148, 1792 // 16, 16), (148, 32, 32), (74, 64, 56), (148, 256, 64), (8, 4, 2)]
    for _ in range(400):
        tiles = rng.randint(1, 600)
        ks = rng.choice([1, 2, 4, 8, 16, 32, 56, 64, 112, 192])
        P = rng.randint(1, 148)
        cases.append((min(P, tiles * ks), tiles, ks))
    for P, tiles, ks in cases:
        check(P, tiles, ks)


def test_one_tile_per_cta_splits_nothing():
    # the whole-tile schedule: as many CTAs as tiles
    for tiles in (104, 112, 128, 148):
        for ks in (16, 32, 56):
            assert all(r[3] == "whole" for mine in roles(tiles, tiles, ks) for r in mine)
