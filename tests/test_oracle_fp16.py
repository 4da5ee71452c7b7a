"""Pins the oracle's own binary16 conversions against numpy's (a library
routine: IEEE 754 binary16, round to nearest even)."""
import numpy as np

import oracle


def test_half_to_float_all_patterns():
    lib = oracle._load()
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float32)
    got = np.array([lib.oracle_half_to_float(int(b)) for b in bits], dtype=np.float32)
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite].view(np.uint32), ref[finite].view(np.uint32))
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(np.isinf(got), np.isinf(ref))


def _float_cases(rng):
    # every binade from below the smallest subnormal half to beyond overflow,
    # each with random mantissas plus the exact ties and their neighbours
    cases = []
    for e in range(-30, 18):
        base = np.float32(2.0) ** e
        mant = rng.integers(0, 1 << 23, size=300).astype(np.uint32)
        x = ((np.uint32(e + 127) << 23) | mant).view(np.float32) if -126 <= e <= 127 else base * (1 + mant / 2**23)
        cases.append(np.asarray(x, np.float32))
        # halfway points between adjacent halves in this binade
        h = np.arange(0, 1024, 7, dtype=np.float64)
        if e >= -14:
            step = 2.0 ** (e - 10)
        else:
            step = 2.0 ** -24
        ties = (base.astype(np.float64) + (h + 0.5) * step).astype(np.float32)
        cases += [ties, np.nextafter(ties, np.float32(0)), np.nextafter(ties, np.float32(np.inf))]
    special = np.array([0.0, 65504.0, 65519.996, 65520.0, 65536.0, 1e30, 6.1035156e-05,
                        5.9604645e-08, 2.9802322e-08, 2.9802326e-08, 8.940697e-08, 1e-40],
                       dtype=np.float32)
    cases.append(special)
    x = np.concatenate(cases)
    return np.concatenate([x, -x])


def test_float_to_half_matches_numpy():
    lib = oracle._load()
    x = _float_cases(np.random.default_rng(1))
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    got = np.array([lib.oracle_float_to_half_rn(float(v)) for v in x], dtype=np.uint16)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(x[i]), hex(got[i]), hex(ref[i])) for i in bad[:10]]


def test_float_to_half_nan_inf():
    assert oracle.float_to_half_bits(float("inf")) == 0x7C00
    assert oracle.float_to_half_bits(float("-inf")) == 0xFC00
    h = oracle.float_to_half_bits(float("nan"))
    assert (h & 0x7C00) == 0x7C00 and (h & 0x3FF) != 0
