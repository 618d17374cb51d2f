"""Pins for the oracle's chunked prefill (``attention_prefill_chunk``).

A chunk is a piece of the prompt: its outputs are fixed by the whole-prompt
prefill (pinned in test_oracle.py) and, for one-token chunks, by the decode
step.  The pins check exactly that, per sequence with different cached
prefixes and with a window, plus a one-hot probe that counts the visible keys
of every chunk row by brute force.
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


def draw(B, N, H, Hkv, D, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, N, H, D)), rng.standard_normal((B, N, Hkv, D)),
            rng.standard_normal((B, N, Hkv, D)), rng.uniform(0.5, 1.5, D))


@pytest.mark.parametrize("over", [dict(), dict(window=5, softcap=20.0),
                                  dict(k_eq_v=True, rotary_fraction=0.5, qk_norm=O.NORM_W),
                                  dict(qk_norm=O.NORM_ONE_PLUS_W, window=40)])
def test_chunk_equals_rows_of_whole_prompt(over):
    c = cfg(**over)
    B, C, Lmax = 3, 7, 40
    prefix = np.array([0, 11, 33])
    q_all, k, v, w = draw(B, Lmax, 4, 2, 16, seed=1)
    wq = wk = w if c["qk_norm"] else None
    q = np.stack([q_all[b, prefix[b]:prefix[b] + C] for b in range(B)])
    got = O.attention_prefill_chunk(q, k, None if c["k_eq_v"] else v, prefix, c, w_q=wq, w_k=wk)
    for b in range(B):
        n = prefix[b] + C
        full = O.attention_prefill(q_all[b:b + 1, :n], k[b:b + 1, :n], None if c["k_eq_v"] else v[b:b + 1, :n],
                                   np.arange(n)[None], c, w_q=wq, w_k=wk)
        assert np.allclose(got[b], full[0, prefix[b]:], rtol=1e-12, atol=1e-12), b


def test_one_token_chunk_equals_decode():
    c = cfg(window=9, softcap=30.0)
    B, Lmax = 2, 30
    q_all, k, v, _ = draw(B, Lmax, 4, 2, 16, seed=2)
    prefix = np.array([4, 21])
    q = np.stack([q_all[b, prefix[b]:prefix[b] + 1] for b in range(B)])
    got = O.attention_prefill_chunk(q, k, v, prefix, c)
    dec = O.attention_decode(q[:, 0], k, v, prefix + 1, c)
    assert np.allclose(got[:, 0], dec, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("W", [0, 6])
def test_chunk_onehot_counts(W):
    # q = 0: uniform weights on the visible keys; one-hot values count them
    c = cfg(num_heads=1, num_kv_heads=1, head_dim=32, window=W)
    Lmax, C, P = 32, 9, 13
    q = np.zeros((1, C, 1, 32))
    k = np.random.default_rng(3).standard_normal((1, Lmax, 1, 32))
    v = np.zeros((1, Lmax, 1, 32))
    v[0, np.arange(Lmax), 0, np.arange(Lmax)] = 1.0
    got = O.attention_prefill_chunk(q, k, v, np.array([P]), c)[0, :, 0]
    for i in range(C):
        t = P + i                                      # the row's token index
        first = 0 if W == 0 else max(0, t - W + 1)
        vis = np.zeros(32, dtype=bool)
        vis[first:t + 1] = True
        assert np.array_equal(got[i] > 0, vis), i
        assert np.allclose(got[i][vis], 1.0 / vis.sum())
