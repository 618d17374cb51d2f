"""Randomised invariants of the oracle (hypothesis, bounded example counts).

The fixed pins in the other oracle tests choose their shapes; these draw them:
any split of a prompt into a cached prefix and a chunk reproduces the whole
prompt's rows, any left padding reproduces the sequence alone, constant values
come back exactly whatever the mask, and the int8 round trip stays within half a
step for any row.
"""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle as O

FAST = settings(max_examples=25, deadline=None)


def cfg(window, softcap, norm, frac):
    return dict(num_heads=2, num_kv_heads=1, head_dim=8, window=window, rope_theta=1e4, rotary_fraction=frac,
                rope_freq_dim=0, softcap=softcap, scalar=8.0, k_eq_v=False, qk_norm=norm, norm_eps=1e-6)


layers = st.builds(cfg, st.sampled_from([0, 1, 3, 9]), st.sampled_from([0.0, 5.0]),
                   st.sampled_from([O.NORM_NONE, O.NORM_W, O.NORM_ONE_PLUS_W]), st.sampled_from([0.0, 0.5, 1.0]))


def draw(seed, n):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((1, n, 2, 8)), rng.standard_normal((1, n, 1, 8)), rng.standard_normal((1, n, 1, 8)),
            rng.uniform(0.5, 1.5, 8))


@FAST
@given(layers, st.integers(1, 20), st.integers(0, 20), st.integers(0, 10_000))
def test_any_chunk_split_reproduces_the_prompt(c, C, P, seed):
    q, k, v, w = draw(seed, P + C)
    wk = w if c["qk_norm"] else None
    got = O.attention_prefill_chunk(q[:, P:], k, v, [P], c, w_q=wk, w_k=wk)
    full = O.attention_prefill(q, k, v, np.arange(P + C)[None], c, w_q=wk, w_k=wk)
    assert np.allclose(got, full[:, P:], rtol=1e-10, atol=1e-12)


@FAST
@given(layers, st.integers(1, 20), st.integers(0, 15), st.integers(0, 10_000))
def test_any_left_padding_reproduces_the_sequence(c, n, pad, seed):
    q, k, v, w = draw(seed, n + pad)
    wk = w if c["qk_norm"] else None
    pos = np.concatenate([np.zeros(pad, dtype=np.int64), np.arange(n)])[None]
    got = O.attention_prefill(q, k, v, pos, c, w_q=wk, w_k=wk, seq_range=[(pad, n + pad)])
    alone = O.attention_prefill(q[:, pad:], k[:, pad:], v[:, pad:], np.arange(n)[None], c, w_q=wk, w_k=wk)
    assert np.allclose(got[:, pad:], alone, rtol=1e-10, atol=1e-12)
    assert np.all(got[:, :pad] == 0)


@FAST
@given(layers, st.integers(1, 25), st.floats(-3.0, 3.0), st.integers(0, 10_000))
def test_constant_values_come_back_exactly(c, n, value, seed):
    q, k, _, w = draw(seed, n)
    wk = w if c["qk_norm"] else None
    v = np.full((1, n, 1, 8), value)
    out = O.attention_prefill(q, k, v, np.arange(n)[None], c, w_q=wk, w_k=wk)
    assert np.allclose(out, value, rtol=1e-12, atol=1e-12)


@FAST
@given(st.integers(1, 64), st.floats(1e-6, 1e6), st.integers(0, 10_000))
def test_int8_round_trip_within_half_step(D, scale, seed):
    x = (np.random.default_rng(seed).standard_normal((3, D)) * scale).astype(np.float32)
    c, s = O.kv_quantize(x)
    err = np.abs(O.kv_dequantize(c, s) - x.astype(np.float64))
    assert np.all(err <= 0.5 * s[:, None].astype(np.float64) * (1 + 1e-6))
    assert np.all(np.abs(c.astype(np.int32)).max(axis=1) == 127)
