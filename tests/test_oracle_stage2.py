"""Exhaustive pins of stage 2 (group UINT4 in the INT8 domain).

"QServe: Low Bit Width Does Not Guarantee High Throughput", section 4: the
stage-2 equation and the protective range [-119,119], which exists so that
the INT4 -> INT8 dequantization (multiply by the integer scale, subtract the
zero compensation) stays inside INT8 and can run lane-parallel in registers.
Every (min, max) pair a group can have is enumerated, with every value in
between.
"""
import numpy as np

import oracle


def _all_groups():
    for mn in range(-119, 1):
        for mx in range(0, 120):
            yield mn, mx, np.arange(mn, mx + 1, dtype=np.int8)


def test_stage2_exhaustive_invariants():
    lanes_ok = True
    for mn, mx, w in _all_groups():
        q, sg, z, zs = oracle.stage2_group(w)
        # integer scale in [1, 16]; zero point is a valid UINT4
        assert 1 <= sg <= 16
        assert 0 <= z <= 15
        assert zs == z * sg
        # the 16-level grid covers the group's range, and no smaller scale does
        assert 15 * sg >= mx - mn
        assert sg == 1 or 15 * (sg - 1) < mx - mn
        # every emitted code is UINT4 and dequantizes inside INT8 without overflow
        assert q.max() <= 15
        what = q.astype(np.int32) * sg - zs
        assert np.abs(what).max() <= 127
        # rounding error at most half a grid step
        assert np.all(2 * np.abs(what - w.astype(np.int32)) <= sg)
        # q is a nearest grid point to w (every alternative code is no closer)
        grid = (np.arange(16)[None, :] - z) * sg
        best = np.abs(grid - w.astype(np.int32)[:, None]).min(axis=1)
        assert np.array_equal(np.abs(what - w), best)
        # byte lanes: the products q*s_g and zs fit an unsigned byte for every
        # q in [0,15], so four lanes of a 32-bit register never carry
        lanes_ok &= (15 * sg <= 240) and (zs <= 240)
    assert lanes_ok


def test_zero_group_and_single_values():
    q, sg, z, zs = oracle.stage2_group(np.zeros(128, np.int8))
    assert (sg, z, zs) == (1, 0, 0) and not q.any()
    for v in (-119, -15, -1, 1, 15, 119):
        g = np.full(128, v, np.int8)
        q, sg, z, zs = oracle.stage2_group(g)
        what = q.astype(int) * sg - zs
        # the range always includes 0, so a constant group is exact only
        # while |v| <= 15 (scale 1); beyond that it is within half a step
        if abs(v) <= 15:
            assert sg == 1 and np.all(what == v)
        assert np.all(2 * np.abs(what - v) <= sg)


def test_multiply_then_subtract_identity():
    """q*s_g - z*s_g == (q - z)*s_g for every UINT4 q and every valid (s_g, z)."""
    qs = np.arange(16, dtype=np.uint8)
    for sg in range(1, 17):
        for z in range(16):
            q = qs[None, :].copy()
            vals = (qs.astype(int) - z) * sg
            ok = (vals >= -128) & (vals <= 127)
            sgt = np.full((1, 1), sg, np.uint8)
            zst = np.full((1, 1), z * sg, np.uint8)
            got = oracle.dequant_weights(q, sgt, zst, 16)[0].astype(int)
            assert np.array_equal(got[ok], vals[ok])


def test_round_half_even_division():
    from fractions import Fraction
    for a in range(-130, 131):
        for b in range(1, 17):
            fr = Fraction(a, b)
            r = oracle.div_round_half_even(a, b)
            assert abs(fr - r) <= Fraction(1, 2)
            if abs(fr - r) == Fraction(1, 2):
                assert r % 2 == 0
