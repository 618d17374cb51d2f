"""Pins for the oracle's transformed-key caches (``keys_transformed``, ``transform_keys``).

A cache may hold the keys after QK-norm and RoPE (each cached key rotated at its
own position) instead of the raw keys.  Attention over such a cache must equal
attention over the raw cache, which test_oracle.py and test_oracle_chunk.py pin;
these tests check exactly that, for decode, chunks and the int8 form.
"""
import numpy as np
import pytest

import oracle as O


def cfg(**kw):
    base = dict(num_heads=4, num_kv_heads=2, head_dim=16, window=0, rope_theta=1e4,
                rotary_fraction=1.0, rope_freq_dim=0, softcap=0.0, scalar=16.0,
                k_eq_v=False, qk_norm=O.NORM_NONE, norm_eps=1e-6)
    base.update(kw)
    return base


LAYERS = [dict(), dict(qk_norm=O.NORM_W, window=7), dict(qk_norm=O.NORM_ONE_PLUS_W, rotary_fraction=0.5,
                                                          softcap=20.0)]


def draw(seed, B=2, L=30):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, 4, 16)), rng.standard_normal((B, L, 2, 16)), rng.standard_normal((B, L, 2, 16)),
            rng.uniform(0.5, 1.5, 16))


@pytest.mark.parametrize("over", LAYERS)
def test_decode_over_transformed_keys_equals_raw(over):
    c = cfg(**over)
    q, k, v, w = draw(1)
    wk = w if c["qk_norm"] else None
    lens = np.array([30, 11])
    kt = np.stack([O.transform_keys(k[b], np.arange(30), c, w_k=wk) for b in range(2)])
    got = O.attention_decode(q, kt, v, lens, c, w_q=wk, w_k=wk, keys_transformed=True)
    ref = O.attention_decode(q, k, v, lens, c, w_q=wk, w_k=wk)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("over", LAYERS)
def test_chunk_over_transformed_keys_equals_raw(over):
    c = cfg(**over)
    _, k, v, w = draw(2, L=40)
    wk = w if c["qk_norm"] else None
    q = np.random.default_rng(3).standard_normal((2, 9, 4, 16))
    pre = np.array([0, 23])
    kt = np.stack([O.transform_keys(k[b], np.arange(40), c, w_k=wk) for b in range(2)])
    got = O.attention_prefill_chunk(q, kt, v, pre, c, w_q=wk, w_k=wk, keys_transformed=True)
    ref = O.attention_prefill_chunk(q, k, v, pre, c, w_q=wk, w_k=wk)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_int8_over_transformed_keys():
    c = cfg(qk_norm=O.NORM_W)
    q, k, v, w = draw(4)
    lens = np.array([30, 5])
    kt = np.stack([O.transform_keys(k[b], np.arange(30), c, w_k=w) for b in range(2)])
    kc, ks = O.kv_quantize(kt)
    vc, vs = O.kv_quantize(v)
    got = O.attention_decode_int8(q, kc, ks, vc, vs, lens, c, w_q=w, w_k=w, keys_transformed=True)
    ref = O.attention_decode(q, O.kv_dequantize(kc, ks), O.kv_dequantize(vc, vs), lens, c, w_q=w, w_k=w,
                             keys_transformed=True)
    assert np.array_equal(got, ref)


def test_tied_values_refuse_transformed_keys():
    c = cfg(k_eq_v=True)
    q, k, _, _ = draw(5)
    with pytest.raises(AssertionError):
        O.attention_decode(q, k, None, np.array([30, 30]), c, keys_transformed=True)
