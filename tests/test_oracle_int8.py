"""Pins for the oracle's int8 KV cache (``kv_quantize``, ``attention_decode_int8``).

The format is a reading (per-row symmetric codes in [-127, 127] with one fp32
scale, max|x| mapped to 127, round half to even): the Atlas "Gemma 4" summary
only says int8 KV caching is offered.  The pins check it against what fixes it
independently of the oracle's code: rows that are exactly codes times a power
of two come back unchanged; every code is a nearest integer to x / s (brute
force over all 255 codes, ties to even on exact halves); the round trip is
within half a step; dequantisation is exact, so an int8 decode over a
representable cache equals the float decode over the same values; and the
output is linear in the value scales.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle as O


def cfg(**kw):
    base = dict(num_heads=2, num_kv_heads=1, head_dim=8, window=0, rope_theta=1e4,
                rotary_fraction=1.0, rope_freq_dim=0, softcap=0.0, scalar=8.0,
                k_eq_v=False, qk_norm=O.NORM_NONE, norm_eps=1e-6)
    base.update(kw)
    return base


def representable(shape, seed):
    """Rows c * 2^e with integer codes |c| <= 127, one code of each row at +-127."""
    rng = np.random.default_rng(seed)
    c = rng.integers(-127, 128, size=shape)
    flat = c.reshape(-1, shape[-1])
    pick = rng.integers(0, shape[-1], size=flat.shape[0])
    flat[np.arange(flat.shape[0]), pick] = rng.choice([-127, 127], size=flat.shape[0])
    e = rng.integers(-20, 6, size=shape[:-1])
    return c.astype(np.int8), np.ldexp(1.0, e).astype(np.float32)


def test_exact_on_codes_times_power_of_two():
    c, s = representable((6, 3, 64), seed=1)
    x = c.astype(np.float64) * s[..., None].astype(np.float64)
    cq, sq = O.kv_quantize(x)
    assert cq.dtype == np.int8 and sq.dtype == np.float32
    assert np.array_equal(cq, c)
    assert np.array_equal(sq, s)


def test_codes_are_nearest_integers_brute_force():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((20, 16)) * rng.uniform(0.01, 30.0, (20, 1))).astype(np.float32)
    c, s = O.kv_quantize(x)
    cand = np.arange(-127, 128)
    for i in range(x.shape[0]):
        si = Fraction(float(s[i]))
        for j in range(x.shape[1]):
            xi = Fraction(float(x[i, j]))
            d = [abs(xi / si - int(k)) for k in cand]
            best = min(d)
            # the code is a nearest integer (up to the float32 rounding of x / s)
            assert abs(d[int(c[i, j]) + 127] - best) <= Fraction(1, 10 ** 5), (i, j)


@pytest.mark.parametrize("vals,codes", [
    ([0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 126.5, 127.0], [0, 2, 2, 0, -2, -2, 126, 127]),
    ([3.5, -3.5, 4.5, 0.25, 0.75, -0.75, 100.5, -127.0], [4, -4, 4, 0, 1, -1, 100, -127]),
])
def test_exact_halves_round_to_even(vals, codes):
    # max|x| = 127 gives s = 1 exactly, so x / s is exact and the ties are true ties
    c, s = O.kv_quantize(np.array([vals]))
    assert s[0] == 1.0
    assert c[0].tolist() == codes


def test_round_trip_within_half_step_and_extremes():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((64, 4, 256)).astype(np.float32)
    x[5, 2] *= 1e-30
    x[6, 1] *= 1e20
    c, s = O.kv_quantize(x)
    back = O.kv_dequantize(c, s)
    err = np.abs(back - x.astype(np.float64))
    assert np.all(err <= 0.5 * s[..., None].astype(np.float64) * (1 + 1e-6))
    assert np.all(np.abs(c.astype(np.int32)) <= 127)
    # the largest magnitude of every row is +-127
    assert np.all(np.max(np.abs(c.astype(np.int32)), axis=-1) == 127)
    # and s * 127 is max|x| to float32 rounding
    amax = np.max(np.abs(x), axis=-1).astype(np.float64)
    assert np.all(np.abs(s.astype(np.float64) * 127.0 - amax) <= amax * 2.0 ** -22)


def test_zero_row():
    c, s = O.kv_quantize(np.zeros((2, 8)))
    assert np.all(c == 0) and np.all(s == 0)
    assert np.all(O.kv_dequantize(c, s) == 0)


def decode_case(k_eq_v=False, qk_norm=O.NORM_NONE, window=0, seed=5):
    B, L, Hkv, D, H = 2, 40, 1, 8, 2
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, D))
    kc, ks = representable((B, L, Hkv, D), seed + 1)
    vc, vs = representable((B, L, Hkv, D), seed + 2)
    lens = np.array([L, 23])
    w = None if qk_norm == O.NORM_NONE else rng.uniform(0.5, 1.5, D)
    c = cfg(k_eq_v=k_eq_v, qk_norm=qk_norm, window=window)
    return q, kc, ks, vc, vs, lens, w, c


@pytest.mark.parametrize("k_eq_v,qk_norm,window", [(False, O.NORM_NONE, 0), (True, O.NORM_W, 0),
                                                    (False, O.NORM_ONE_PLUS_W, 9)])
def test_int8_decode_equals_float_decode_on_representable_cache(k_eq_v, qk_norm, window):
    q, kc, ks, vc, vs, lens, w, c = decode_case(k_eq_v, qk_norm, window)
    kf = kc.astype(np.float64) * ks[..., None]
    vf = vc.astype(np.float64) * vs[..., None]
    got = O.attention_decode_int8(q, kc, ks, vc, vs, lens, c, w_q=w, w_k=w)
    ref = O.attention_decode(q, kf, None if k_eq_v else vf, lens, c, w_q=w, w_k=w)
    assert np.array_equal(got, ref)


def test_int8_output_is_linear_in_value_scales():
    q, kc, ks, vc, vs, lens, w, c = decode_case(seed=9)
    a = O.attention_decode_int8(q, kc, ks, vc, vs, lens, c)
    b = O.attention_decode_int8(q, kc, ks, vc, vs * np.float32(4.0), lens, c)
    assert np.allclose(b, 4.0 * a, rtol=1e-12, atol=0)
    # the key scales move the weights, not the scale of the output
    k2 = O.attention_decode_int8(q, kc, ks * np.float32(0.0), vc, vs, lens, c)
    vals = vc.astype(np.float64) * vs[..., None]
    for b_ in range(2):
        mean_v = vals[b_, :lens[b_], 0].mean(axis=0)        # all logits 0: uniform weights
        assert np.allclose(k2[b_, 0], mean_v, rtol=1e-12, atol=1e-300)


def test_int8_keqv_ignores_value_arrays():
    q, kc, ks, vc, vs, lens, w, c = decode_case(k_eq_v=True, seed=11)
    a = O.attention_decode_int8(q, kc, ks, vc, vs, lens, c)
    b = O.attention_decode_int8(q, kc, ks, -vc, vs * 3, lens, c)
    assert np.array_equal(a, b)


def test_int8_decode_close_to_unquantised():
    # a quantised N(0, 1) cache moves the output by about the quantisation step
    rng = np.random.default_rng(13)
    B, L, D = 1, 300, 64
    q = rng.standard_normal((B, 2, D))
    k = rng.standard_normal((B, L, 1, D))
    v = rng.standard_normal((B, L, 1, D))
    c = cfg(head_dim=D, scalar=float(D))
    kc, ks = O.kv_quantize(k)
    vc, vs = O.kv_quantize(v)
    lens = np.array([L])
    got = O.attention_decode_int8(q, kc, ks, vc, vs, lens, c)
    ref = O.attention_decode(q, k, v, lens, c)
    step = float(np.max(vs))
    assert np.max(np.abs(got - ref)) < 2 * step
