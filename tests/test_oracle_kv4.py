"""Pins of the oracle's KV4 decode attention with SmoothAttention.

The pages ("QServe: Low Bit Width Does Not Guarantee High Throughput",
section 4; "QServe Guide: W4A8KV4 Quantization for LLM Serving", The
Architecture, subsection 3) define the smoothing (K' = K / lambda, Q' = Q *
lambda, lambda = max|K|^alpha, alpha = 0.5) and 4-bit KV with per-channel
scales; they print no worked example.  The oracle is pinned here against:
the textbook attention of the unquantized inputs within the error bound the
4-bit grid implies; closed forms (uniform and one-hot softmax, one token);
numpy's own IEEE arithmetic for the quantizer; and the smoothing identity.
"""
import numpy as np
import pytest

import oracle


def _rng(s):
    return np.random.default_rng(s)


def _f(x):
    return np.asarray(x).view(np.float16).astype(np.float64)


def _case(seed, Hq=4, Hkv=2, L=96, d=64, k_outlier=25.0):
    r = _rng(seed)
    K = r.standard_normal((Hkv, L, d))
    K[:, :, 5] *= k_outlier          # an outlier key channel, as the guide's illustration injects
    V = r.standard_normal((Hkv, L, d))
    q = r.standard_normal((Hq, d))
    return q.astype(np.float16), K.astype(np.float16), V.astype(np.float16)


def _exact_attention(q, K, V):
    """Textbook attention of the unquantized FP16 inputs, binary64."""
    Hq, d = q.shape
    Hkv = K.shape[0]
    G = Hq // Hkv
    out = np.zeros((Hq, d))
    for h in range(Hq):
        g = h // G
        s = K[g].astype(np.float64) @ q[h].astype(np.float64) / np.sqrt(d)
        p = np.exp(s - s.max())
        p /= p.sum()
        out[h] = p @ V[g].astype(np.float64)
    return out


def test_lambda_is_sqrt_of_channel_max():
    q, K, V = _case(1)
    lam = oracle.smooth_lambda(K[0])
    want = np.maximum(np.sqrt(np.abs(K[0].astype(np.float64)).max(axis=0)), 1e-5).astype(np.float16)
    assert np.array_equal(lam, want.view(np.uint16))
    zero = np.zeros((8, 16), np.float16)
    assert np.all(_f(oracle.smooth_lambda(zero)) == np.float64(np.float16(1e-5)))


def test_quantizer_matches_numpy_and_its_bound():
    q, K, V = _case(2)
    lam = oracle.smooth_lambda(K[0])
    codes, s = oracle.kv4_quantize(K[0], lam)
    xs = K[0].astype(np.float32) / _f(lam).astype(np.float32)
    sw = (np.abs(xs).max(axis=0) / np.float32(7.0)).astype(np.float16)
    assert np.array_equal(s, sw.view(np.uint16))
    want = np.clip(np.rint(xs / sw.astype(np.float32)), -8, 7).astype(np.int8)
    assert np.array_equal(codes, want)
    err = np.abs(codes * _f(s) - xs)
    inside = np.abs(codes) < 7
    assert np.all(err[inside] <= _f(s)[None, :].repeat(len(xs), 0)[inside] / 2 + 1e-6)
    assert codes.min() >= -8 and codes.max() <= 7


def test_smoothing_flattens_the_outlier_channel():
    q, K, V = _case(3)
    lam = oracle.smooth_lambda(K[0])
    xs = K[0].astype(np.float64) / _f(lam)
    # the outlier channel's range shrinks from ~25x the others to ~sqrt(25)x
    ratio_before = np.abs(K[0][:, 5].astype(float)).max() / np.abs(np.delete(K[0], 5, 1).astype(float)).max()
    ratio_after = np.abs(xs[:, 5]).max() / np.abs(np.delete(xs, 5, 1)).max()
    assert ratio_after < ratio_before / 3


@pytest.mark.parametrize("seed", [4, 5, 6])
def test_close_to_textbook_attention_within_the_grid_bound(seed):
    q, K, V = _case(seed)
    r = oracle.kv4_decode(q, K, V)
    got = _f(r["out"]).reshape(q.shape)
    exact = _exact_attention(q, K, V)
    Hq, d = q.shape
    G = Hq // K.shape[0]
    for h in range(Hq):
        g = h // G
        lam, sk, sv = _f(r["lam"][g]), _f(r["s_k"][g]), _f(r["s_v"][g])
        # score error <= sum_c |q lam| s_k / 2 / sqrt(d); softmax ratio error <= 2x that
        ek = np.sum(np.abs(q[h].astype(float) * lam) * sk) / 2 / np.sqrt(d)
        bound = (np.exp(2 * ek) - 1) * np.abs(V[g].astype(float)).max(axis=0) + sv / 2 \
            + np.spacing(np.abs(exact[h]).astype(np.float16)).astype(float)
        assert np.all(np.abs(got[h] - exact[h]) <= bound), h


def test_dropping_lambda_from_the_query_breaks_the_bound():
    """A plausible mistake (smoothing the keys but not the query) is caught
    by the same bound."""
    q, K, V = _case(7)
    r = oracle.kv4_decode(q, K, V)
    ones = np.full_like(r["lam"], np.float16(1.0).view(np.uint16))
    bad = _f(oracle.kv4_attention(q, r["k_codes"], r["s_k"], r["v_codes"], r["s_v"], ones)).reshape(q.shape)
    exact = _exact_attention(q, K, V)
    assert np.abs(bad - exact).max() > 0.1


def test_uniform_softmax_gives_the_mean_of_the_values():
    r = _rng(8)
    Hq, Hkv, L, d = 2, 1, 40, 32
    q = r.standard_normal((Hq, d)).astype(np.float16)
    codes_k = np.zeros((Hkv, L, d), np.int8)                  # all scores equal
    codes_v = r.integers(-8, 8, (Hkv, L, d)).astype(np.int8)
    s = np.full((Hkv, d), np.float16(0.25)).view(np.uint16)
    lam = np.full((Hkv, d), np.float16(1.0)).view(np.uint16)
    out = _f(oracle.kv4_attention(q, codes_k, s, codes_v, s, lam)).reshape(Hq, d)
    want = (codes_v[0].astype(float) * 0.25).mean(axis=0).astype(np.float16).astype(float)
    assert np.array_equal(out[0], want) and np.array_equal(out[1], want)


def test_single_token_and_dominant_token():
    r = _rng(9)
    Hq, Hkv, d = 2, 1, 32
    q = np.ones((Hq, d), np.float16)
    s = np.full((Hkv, d), np.float16(0.5)).view(np.uint16)
    lam = np.full((Hkv, d), np.float16(1.0)).view(np.uint16)
    cv = r.integers(-8, 8, (Hkv, 1, d)).astype(np.int8)
    out = _f(oracle.kv4_attention(q, np.full((1, 1, d), 3, np.int8), s, cv, s, lam)).reshape(Hq, d)
    assert np.array_equal(out[0], cv[0, 0] * 0.5)              # L = 1: the one value row
    ck = np.zeros((1, 5, d), np.int8)
    ck[0, 3] = 7                                               # token 3: score 7*0.5*32/sqrt(32) ~ 19.8 above the rest
    cv5 = r.integers(-8, 8, (1, 5, d)).astype(np.int8)
    out = _f(oracle.kv4_attention(q, ck, s, cv5, s, lam)).reshape(Hq, d)
    assert np.allclose(out[0], cv5[0, 3] * 0.5, atol=1e-6 * 8 + 4 * 2.0 ** -11)
