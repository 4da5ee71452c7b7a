"""The per-token quantizer's rounding shortcut, restated in numpy float32
(no GPU): multiply by fl(1/s_x), clamp to [-128, 127], round by adding
1.5 * 2^23, and fall back to the IEEE division only within 2^-12 of a
rounding boundary.  Over every finite FP16 x and a spread of FP16 scales
(subnormal ones included) the shortcut gives clamp(rint(fl(x / s_x))), the
oracle's definition, wherever it does not fall back."""
import numpy as np

MAGIC = np.float32(12582912.0)      # 1.5 * 2^23
FAR = np.float32(0.499755859375)    # 1/2 - 2^-12


def _shortcut(x, sx):
    r = np.float32(1.0) / sx
    c = np.clip((x * r).astype(np.float32), np.float32(-128.0), np.float32(127.0)).astype(np.float32)
    y = (c + MAGIC).astype(np.float32)
    near = np.abs((c - (y - MAGIC).astype(np.float32)).astype(np.float32)) >= FAR
    code = (y.view(np.uint32) & 0xFF).astype(np.uint8).view(np.int8).astype(np.int32)
    return code, near


def test_shortcut_equals_division():
    xs = np.arange(65536, dtype=np.uint32).astype(np.uint16).view(np.float16)
    xs = xs[np.isfinite(xs)].astype(np.float32)
    scales = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float32)
    rng = np.random.default_rng(7)
    pick = np.concatenate([scales[:40], scales[-20:], rng.choice(scales, 140, replace=False),
                           np.float32([1.0, 0.5, 1.0 / 127.0, 3.3 / 127.0])])
    fell_back = 0
    for sx in pick.astype(np.float32):
        code, near = _shortcut(xs, sx)
        exact = np.clip(np.rint((xs / sx).astype(np.float32)), -128, 127).astype(np.int32)
        assert np.array_equal(code[~near], exact[~near])
        fell_back += int(near.sum())
    # the fallback is rare: well under 1 in 1000 elements
    assert fell_back < 1e-3 * xs.size * pick.size


def test_ties_take_the_division_and_the_clamp_decides_beyond_the_range():
    sx = np.float32(1.0)
    x = np.float32([0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 126.5, -127.5, 127.5, -128.5])
    code, near = _shortcut(x, sx)
    assert near[:8].all()              # exact ties always take the division
    assert list(code[8:]) == [127, -128] and not near[8:].any()   # the clamp decides
