"""Pins for the float64 oracle: closed forms, invariants, brute force and a
library routine -- nothing here re-evaluates the oracle's own formulas.

Each test names what the model cards fix and what it checks.  A plausible
slip in the oracle (a dropped gain, a wrong rotation sign or pairing, an
off-by-one window, a transposed head mapping, V taken after the norm) fails at
least one of them; ``test_planted_mistakes_are_caught`` plants such slips in a
copy of the oracle and checks exactly that.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def layer(**kw):
    base = dict(num_heads=1, num_kv_heads=1, head_dim=2, window=0, rope_theta=1e4,
                rotary_fraction=0.0, rope_freq_dim=0, softcap=0.0, scalar=1.0,
                k_eq_v=False, qk_norm=O.NORM_NONE, norm_eps=1e-6)
    base.update(kw)
    return base


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# --- softcap: c*tanh(x/c) (ZeroModels "Gemma 2", logit softcapping bullet) ----

def test_softcap_closed_form():
    c = 50.0
    tanh1, tanh10 = 0.7615941559557649, 0.9999999958776927  # tabulated tanh(1), tanh(10)
    assert O.softcap(0.0, c) == 0.0
    assert O.softcap(c, c) == pytest.approx(c * tanh1, rel=1e-15)
    assert O.softcap(-c, c) == pytest.approx(-c * tanh1, rel=1e-15)
    assert O.softcap(10 * c, c) == pytest.approx(c * tanh10, rel=1e-15)
    # Taylor: x - x^3/(3c^2) for |x| << c
    x = 1e-3
    assert O.softcap(x, c) == pytest.approx(x - x ** 3 / (3 * c * c), rel=1e-15)
    # bounded, odd, monotone
    xs = np.linspace(-1e4, 1e4, 2001)
    ys = O.softcap(xs, c)
    assert np.all(np.abs(ys) <= c) and np.all(np.diff(ys) >= 0)
    assert np.array_equal(O.softcap(-xs, c), -ys)
    # no cap: c <= 0 is the identity; a huge cap is the identity to 1e-12
    assert np.array_equal(O.softcap(xs, 0.0), xs)
    assert np.max(np.abs(O.softcap(xs, 1e30) - xs)) < 1e-12


def test_softcap_huge_equals_no_softcap_in_layer():
    S, D = 9, 8
    q, k, v = rnd((1, S, 2, D), 1) * 4, rnd((1, S, 1, D), 2) * 4, rnd((1, S, 1, D), 3)
    pos = np.arange(S)[None]
    a = O.attention_prefill(q, k, v, pos, layer(num_heads=2, head_dim=D, softcap=1e30))
    b = O.attention_prefill(q, k, v, pos, layer(num_heads=2, head_dim=D, softcap=0.0))
    assert np.max(np.abs(a - b)) < 1e-12


# --- RMSNorm (KerasFormers "Gemma 4", What changed; norm_eps 1e-6) -------------

def test_rms_norm_worked_example():
    # x = (3, 4): mean square 12.5, so x / sqrt(12.5) = (0.6*sqrt2, 0.8*sqrt2)
    x = np.array([3.0, 4.0])
    out = O.rms_norm(x, np.ones(2), O.NORM_W, 0.0)
    assert out == pytest.approx([0.6 * math.sqrt(2), 0.8 * math.sqrt(2)], rel=1e-15)
    out1 = O.rms_norm(x, np.zeros(2), O.NORM_ONE_PLUS_W, 0.0)
    assert np.array_equal(out, out1)
    # eps enters under the root: sqrt(12.5 + 0.5) = sqrt(13)
    out_e = O.rms_norm(x, np.ones(2), O.NORM_W, 0.5)
    assert out_e == pytest.approx([3 / math.sqrt(13), 4 / math.sqrt(13)], rel=1e-15)
    # the gain multiplies per dimension
    g = np.array([2.0, -0.5])
    assert O.rms_norm(x, g, O.NORM_W, 0.0) == pytest.approx(out * g, rel=1e-15)


def test_rms_norm_invariants():
    x = rnd((5, 7, 64), 4)
    w = rnd(64, 5) * 0.1
    y = O.rms_norm(x, np.ones(64), O.NORM_W, 0.0)
    assert np.max(np.abs(np.sqrt(np.mean(y * y, axis=-1)) - 1.0)) < 1e-14
    # Gemma's (1 + w) gain is the plain gain at w + 1, exactly
    assert np.array_equal(O.rms_norm(x, w, O.NORM_ONE_PLUS_W, 1e-6),
                          O.rms_norm(x, w + 1.0, O.NORM_W, 1e-6))
    # scale invariant for eps = 0
    assert np.max(np.abs(O.rms_norm(7.5 * x, w, O.NORM_W, 0.0) -
                         O.rms_norm(x, w, O.NORM_W, 0.0))) < 1e-13
    # mode none is the identity
    assert np.array_equal(O.rms_norm(x, None, O.NORM_NONE, 1e-6), x)


# --- RoPE (KerasFormers "Gemma 3" dual bases; "Gemma 4" partial rotation) ------

def test_rope_worked_example():
    # D = R = F = 4, theta 1e4: pair (0,2) turns by pos*1, pair (1,3) by pos*0.01
    x = np.array([1.0, 1.0, 0.0, 0.0])
    y = O.rope(x, np.array(1.0), 4, 1e4, 4)
    cos1, sin1 = 0.5403023058681398, 0.8414709848078965        # tabulated
    cos01, sin01 = 0.9999500004166653, 0.009999833334166664    # tabulated
    assert y == pytest.approx([cos1, cos01, sin1, sin01], rel=1e-15)
    # the second element of each pair turns the other way round
    y2 = O.rope(np.array([0.0, 0.0, 1.0, 1.0]), np.array(1.0), 4, 1e4, 4)
    assert y2 == pytest.approx([-sin1, -sin01, cos1, cos01], rel=1e-15)


def test_rope_is_complex_rotation():
    # textbook form: (x_t + i x_{t+R/2}) * exp(i pos theta^(-2t/F))
    D, R, F, theta = 64, 64, 64, 1e6
    x = rnd((10, D), 6)
    pos = np.arange(10) * 997.0
    y = O.rope(x, pos[:, None][:, 0], R, theta, F)
    z = (x[:, :R // 2] + 1j * x[:, R // 2:R]) * np.exp(
        1j * pos[:, None] * np.power(theta, -np.arange(R // 2) * 2.0 / F))
    assert np.max(np.abs(y[:, :R // 2] - z.real)) < 1e-12
    assert np.max(np.abs(y[:, R // 2:R] - z.imag)) < 1e-12


def test_rope_invariants():
    D = 512
    x = rnd((33, D), 7)
    pos = np.arange(33) * 1000.0
    for R in (512, 128):
        y = O.rope(x, pos, R, 1e6, D)
        assert np.max(np.abs(np.linalg.norm(y, axis=-1) - np.linalg.norm(x, axis=-1))) < 1e-12
        assert np.array_equal(O.rope(x, np.zeros(33), R, 1e6, D), x)
        # dims past the rotated slice are copied bit for bit
        assert np.array_equal(y[:, R:], x[:, R:])
    assert np.array_equal(O.rope(x, pos, 0, 1e6, D), x)


@pytest.mark.parametrize("rot,fd", [(256, 0), (64, 0), (64, 64)])
def test_rope_relative_position(rot, fd):
    # q~(i).k~(j) depends on i-j only: shifting every position leaves the layer unchanged
    S, D = 12, 256
    q, k, v = rnd((1, S, 2, D), 8), rnd((1, S, 1, D), 9), rnd((1, S, 1, D), 10)
    cfg = layer(num_heads=2, head_dim=D, rotary_fraction=rot / D, rope_freq_dim=fd,
                scalar=D, rope_theta=1e4)
    pos = np.arange(S)[None]
    base = O.attention_prefill(q, k, v, pos, cfg)
    for delta in (1, 1000, 30000):
        moved = O.attention_prefill(q, k, v, pos + delta, cfg)
        assert np.max(np.abs(moved - base)) < 1e-9
    # but a position *change of spacing* does change it
    spread = O.attention_prefill(q, k, v, pos * 2, cfg)
    assert np.max(np.abs(spread - base)) > 1e-3


# --- masking (ZeroModels "Gemma 2" alternating attention; Gemma 3/4 windows) ----

def _onehot_probe(S, W):
    D = max(S, 2)
    q = np.zeros((1, S, 1, D))
    k = rnd((1, S, 1, D), 11)
    v = np.eye(S, D)[None, :, None, :]
    return O.attention_prefill(q, k, v, np.arange(S)[None], layer(head_dim=D, window=W))[0, :, 0]


@pytest.mark.parametrize("S", [1, 2, 3, 7, 12])
def test_mask_onehot_probe_counts(S):
    # q = 0 gives uniform weights over the visible keys; one-hot values read them out.
    # Visible count: min(i+1, W) keys ending at i itself (W = 0: all i+1).
    for W in range(0, S + 3):
        wts = _onehot_probe(S, W)[:, :S]
        for i in range(S):
            n = i + 1 if W == 0 else min(i + 1, W)
            expect = np.zeros(S)
            expect[i - n + 1:i + 1] = 1.0 / n
            assert np.max(np.abs(wts[i] - expect)) < 1e-15, (S, W, i)


def test_mask_window_limits():
    S, D = 10, 16
    q, k, v = rnd((1, S, 2, D), 12), rnd((1, S, 1, D), 13), rnd((1, S, 1, D), 14)
    pos = np.arange(S)[None]
    full = O.attention_prefill(q, k, v, pos, layer(num_heads=2, head_dim=D, window=0))
    for W in (S, S + 1, S + 5):
        assert np.array_equal(O.attention_prefill(q, k, v, pos, layer(num_heads=2, head_dim=D, window=W)), full)
    one = O.attention_prefill(q, k, v, pos, layer(num_heads=2, head_dim=D, window=1))
    assert np.max(np.abs(one[0, :, 0] - v[0, :, 0])) < 1e-15
    assert np.max(np.abs(one[0, :, 1] - v[0, :, 0])) < 1e-15


def test_mask_future_and_past_independence():
    # causal: row i ignores keys/values after i; window W: row i ignores keys before i-W+1
    S, D, W = 11, 8, 4
    q, k, v = rnd((1, S, 1, D), 15), rnd((1, S, 1, D), 16), rnd((1, S, 1, D), 17)
    pos = np.arange(S)[None]
    cfg = layer(head_dim=D, window=W, scalar=D)
    base = O.attention_prefill(q, k, v, pos, cfg)[0, :, 0]
    i = 7
    for j in range(S):
        k2, v2 = k.copy(), v.copy()
        k2[0, j] += 3.0
        v2[0, j] += 3.0
        row = O.attention_prefill(q, k2, v2, pos, cfg)[0, i, 0]
        changed = np.max(np.abs(row - base[i])) > 1e-9
        assert changed == (i - W < j <= i), j


def test_mask_brute_force_loops():
    # literal per-element loops with math.exp (no numpy in the reduction)
    S, D = 6, 3
    q, k, v = rnd((1, S, 1, D), 18), rnd((1, S, 1, D), 19), rnd((1, S, 1, D), 20)
    for W in range(0, S + 2):
        got = O.attention_prefill(q, k, v, np.zeros((1, S)), layer(head_dim=D, window=W))[0, :, 0]
        for i in range(S):
            lo = 0 if W == 0 else max(0, i - W + 1)
            logits = [sum(q[0, i, 0, d] * k[0, j, 0, d] for d in range(D)) for j in range(lo, i + 1)]
            mx = max(logits)
            ex = [math.exp(s - mx) for s in logits]
            den = sum(ex)
            for d in range(D):
                ref = sum(e * v[0, lo + n, 0, d] for n, e in enumerate(ex)) / den
                assert abs(got[i, d] - ref) < 1e-13


# --- the softmax/PV closed form on a 3-token example --------------------------

def test_worked_three_tokens():
    # D=2, no RoPE, scale 1.  q = k = (1,0),(0,1),(1,1); v = (1,2),(3,4),(5,6).
    q = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]])[None, :, None]
    v = np.array([[1.0, 2.0], [3.0, 4.0], [5.0, 6.0]])[None, :, None]
    e = math.e
    row0 = [1.0, 2.0]
    row1 = [(1 + 3 * e) / (1 + e), (2 + 4 * e) / (1 + e)]        # logits (0, 1)
    row2 = [(4 + 5 * e) / (2 + e), (6 + 6 * e) / (2 + e)]        # logits (1, 1, 2)
    got = O.attention_prefill(q, q, v, np.zeros((1, 3)), layer())[0, :, 0]
    assert got == pytest.approx(np.array([row0, row1, row2]), rel=1e-15)
    # window 2: row 2 sees keys 1, 2 with logits (1, 2)
    got_w = O.attention_prefill(q, q, v, np.zeros((1, 3)), layer(window=2))[0, 2, 0]
    assert got_w == pytest.approx([(3 + 5 * e) / (1 + e), (4 + 6 * e) / (1 + e)], rel=1e-15)
    # softcap 1: logits become tanh of themselves
    t1, t2 = 0.7615941559557649, 0.9640275800758169               # tabulated tanh(1), tanh(2)
    a, b = math.exp(t1), math.exp(t2)
    got_c = O.attention_prefill(q, q, v, np.zeros((1, 3)), layer(softcap=1.0))[0, 2, 0]
    assert got_c == pytest.approx([(4 * a + 5 * b) / (2 * a + b), (6 * a + 6 * b) / (2 * a + b)], rel=1e-14)
    # query_pre_attn_scalar 4: scale 1/2 -> row 1 logits (0, 1/2)
    h = math.exp(0.5)
    got_s = O.attention_prefill(q, q, v, np.zeros((1, 3)), layer(scalar=4.0))[0, 1, 0]
    assert got_s == pytest.approx([(1 + 3 * h) / (1 + h), (2 + 4 * h) / (1 + h)], rel=1e-15)


def test_softmax_of_constant_values():
    S, D = 17, 32
    q, k = rnd((2, S, 4, D), 21) * 3, rnd((2, S, 2, D), 22) * 3
    v = np.ones((2, S, 2, D))
    out = O.attention_prefill(q, k, v, np.tile(np.arange(S), (2, 1)),
                              layer(num_heads=4, num_kv_heads=2, head_dim=D, window=5,
                                    softcap=5.0, rotary_fraction=1.0, scalar=D))
    assert np.max(np.abs(out - 1.0)) < 1e-14


# --- textbook reduction: torch SDPA (float64, CPU) ----------------------------

@pytest.mark.parametrize("W", [0, 5])
def test_matches_torch_sdpa(W):
    B, S, H, Hkv, D = 2, 23, 4, 2, 32
    q, k, v = rnd((B, S, H, D), 23), rnd((B, S, Hkv, D), 24), rnd((B, S, Hkv, D), 25)
    pos = np.tile(np.arange(S), (B, 1))
    cfg = layer(num_heads=H, num_kv_heads=Hkv, head_dim=D, window=W, scalar=D, rotary_fraction=1.0)
    got = O.attention_prefill(q, k, v, pos, cfg)
    # rotate with the oracle, then let torch do the attention itself
    qr = torch.from_numpy(O.rope(q, pos[:, :, None], D, 1e4, D)).permute(0, 2, 1, 3)
    kr = torch.from_numpy(O.rope(k, pos[:, :, None], D, 1e4, D)).permute(0, 2, 1, 3)
    vt = torch.from_numpy(v).permute(0, 2, 1, 3)
    kr = kr.repeat_interleave(H // Hkv, dim=1)
    vt = vt.repeat_interleave(H // Hkv, dim=1)
    ones = torch.ones(S, S, dtype=torch.bool)
    band = torch.tril(ones) if W == 0 else torch.tril(ones) & torch.triu(ones, diagonal=-(W - 1))
    ref = torch.nn.functional.scaled_dot_product_attention(qr, kr, vt, attn_mask=band,
                                                           scale=D ** -0.5)
    assert np.max(np.abs(ref.permute(0, 2, 1, 3).numpy() - got)) < 1e-10


# --- K=V, MQA == replicated GQA, decode == last prefill row --------------------

def test_k_eq_v_is_passing_v_equals_k():
    S, D = 13, 64
    q, k = rnd((1, S, 4, D), 26), rnd((1, S, 1, D), 27)
    w = 1.0 + 0.1 * rnd(D, 28)
    kw = dict(num_heads=4, head_dim=D, rotary_fraction=0.25, qk_norm=O.NORM_W, scalar=D)
    pos = np.arange(S)[None]
    a = O.attention_prefill(q, k, None, pos, layer(k_eq_v=True, **kw), w_q=w, w_k=w)
    b = O.attention_prefill(q, k, k, pos, layer(k_eq_v=False, **kw), w_q=w, w_k=w)
    assert np.array_equal(a, b)
    # values are the raw keys, not the normed/rotated ones: with a big gain
    # the normed keys differ from k, and so would the output
    c = O.attention_prefill(q, k, 5.0 * k, pos, layer(k_eq_v=False, **kw), w_q=w, w_k=w)
    assert np.max(np.abs(c - 5.0 * a)) < 1e-12


def test_mqa_equals_replicated_gqa():
    S, H, D = 15, 8, 32
    q, k, v = rnd((2, S, H, D), 29), rnd((2, S, 1, D), 30), rnd((2, S, 1, D), 31)
    pos = np.tile(np.arange(S), (2, 1))
    kw = dict(num_heads=H, head_dim=D, rotary_fraction=1.0, window=6, scalar=D)
    mqa = O.attention_prefill(q, k, v, pos, layer(num_kv_heads=1, **kw))
    rep = O.attention_prefill(q, np.repeat(k, H, axis=2), np.repeat(v, H, axis=2), pos,
                              layer(num_kv_heads=H, **kw))
    assert np.array_equal(mqa, rep)
    # GQA groups are contiguous: heads 0..G-1 read kv head 0
    G = 4
    k2, v2 = rnd((2, S, 2, D), 32), rnd((2, S, 2, D), 33)
    gqa = O.attention_prefill(q, k2, v2, pos, layer(num_kv_heads=2, **kw))
    first = O.attention_prefill(q[:, :, :G], k2[:, :, :1], v2[:, :, :1], pos,
                                layer(**dict(kw, num_heads=G), num_kv_heads=1))
    assert np.array_equal(gqa[:, :, :G], first)


@pytest.mark.parametrize("W,qk", [(0, O.NORM_NONE), (4, O.NORM_ONE_PLUS_W), (0, O.NORM_W)])
def test_decode_equals_last_prefill_row(W, qk):
    B, S, H, Hkv, D = 3, 21, 4, 2, 64
    q, k, v = rnd((B, S, H, D), 34), rnd((B, S, Hkv, D), 35), rnd((B, S, Hkv, D), 36)
    w_q, w_k = 0.1 * rnd(D, 37) + (qk == O.NORM_W), 0.1 * rnd(D, 38) + (qk == O.NORM_W)
    cfg = layer(num_heads=H, num_kv_heads=Hkv, head_dim=D, window=W, rotary_fraction=0.5,
                qk_norm=qk, scalar=D, softcap=3.0)
    pos = np.tile(np.arange(S), (B, 1))
    lens = np.array([S, 9, 1])
    pre = O.attention_prefill(q, k, v, pos, cfg, w_q=w_q, w_k=w_k)
    dq = np.stack([q[b, lens[b] - 1] for b in range(B)])
    dec = O.attention_decode(dq, k, v, lens, cfg, w_q=w_q, w_k=w_k)
    for b in range(B):
        # a prefix of the prompt is itself a prompt
        ref = pre[b, lens[b] - 1] if lens[b] == S else O.attention_prefill(
            q[b:b + 1, :lens[b]], k[b:b + 1, :lens[b]], v[b:b + 1, :lens[b]],
            pos[b:b + 1, :lens[b]], cfg, w_q=w_q, w_k=w_k)[0, -1]
        assert np.max(np.abs(dec[b] - ref)) < 1e-12


@pytest.mark.parametrize("chunk", [1, 7, 64, 200])
def test_split_kv_merge_matches_unsplit(chunk):
    L, D = 200, 16
    s = rnd(L, 39) * 5
    vals = rnd((L, D), 40)
    p = np.exp(s - s.max())
    ref = (p / p.sum()) @ vals
    parts = [O.chunk_partial(s[c:c + chunk], vals[c:c + chunk]) for c in range(0, L, chunk)]
    assert np.max(np.abs(O.lse_merge(parts) - ref)) < 1e-13


# --- the workloads carry the model cards' constants ---------------------------

def test_workloads_use_model_card_constants():
    g = {k: v["value"] for k, v in json.load(open(os.path.join(GOLDEN, "model_card_constants.json"))).items()
         if not k.startswith("_")}
    l1 = W.GEMMA1_MQA.layer
    assert (l1.num_heads, l1.num_kv_heads, l1.head_dim, l1.rope_theta) == (
        g["gemma1_num_heads"], g["gemma1_num_kv_heads"], g["gemma1_head_dim"], g["gemma1_rope_theta"])
    l2 = W.GEMMA2_LOCAL.layer
    assert (l2.num_heads, l2.num_kv_heads, l2.scalar, l2.softcap) == (
        g["gemma2_num_heads"], g["gemma2_num_kv_heads"], g["gemma2_query_pre_attn_scalar"],
        g["gemma2_attn_softcap"])
    l3, l3g = W.GEMMA3_LOCAL.layer, W.GEMMA3_GLOBAL.layer
    assert (l3.num_heads, l3.num_kv_heads, l3.window, l3.rope_theta, l3g.rope_theta, l3.scalar,
            l3.norm_eps) == (g["gemma3_num_heads"], g["gemma3_num_kv_heads"], g["gemma3_sliding_window"],
                             g["gemma3_rope_theta_local"], g["gemma3_rope_theta_global"],
                             g["gemma3_query_pre_attn_scalar"], g["norm_eps"])
    l4, d4l = W.GEMMA4_GLOBAL.layer, W.GEMMA4_DECODE_LOCAL.layer
    assert (l4.num_heads, l4.num_kv_heads, l4.head_dim, l4.rotary_fraction, l4.k_eq_v) == (
        g["gemma4_num_heads"], g["gemma4_num_global_kv_heads"], g["gemma4_global_head_dim"],
        g["gemma4_partial_rotary_factor"], g["gemma4_k_eq_v"])
    assert (d4l.num_kv_heads, d4l.head_dim, d4l.window) == (
        g["gemma4_num_kv_heads"], g["gemma4_head_dim"], g["gemma4_sliding_window"])


# --- padded batches: each sequence's valid tokens [lo, hi) (KerasFormers "Gemma 4",
# Gemma4Generate.generate: attention_mask 1 = keep, 0 = padding) ---------------------

def test_seq_range_full_equals_unpadded():
    B, S, D = 2, 9, 8
    q, k, v = rnd((B, S, 2, D), 40), rnd((B, S, 1, D), 41), rnd((B, S, 1, D), 42)
    pos = np.tile(np.arange(S), (B, 1))
    for W in (0, 3):
        cfg = layer(num_heads=2, head_dim=D, window=W, rotary_fraction=1.0)
        full = O.attention_prefill(q, k, v, pos, cfg)
        rng = np.array([[0, S]] * B)
        assert np.array_equal(O.attention_prefill(q, k, v, pos, cfg, seq_range=rng), full)


@pytest.mark.parametrize("W", [0, 1, 4])
def test_left_padding_equals_sequence_alone(W):
    # a sequence of n tokens placed after S - n padding tokens (garbage values,
    # any positions), with range [S - n, S), gives on its rows what it gives alone
    S, n, D = 11, 7, 8
    x_q, x_k, x_v = rnd((1, n, 2, D), 43), rnd((1, n, 1, D), 44), rnd((1, n, 1, D), 45)
    cfg = layer(num_heads=2, head_dim=D, window=W, rotary_fraction=0.5, rope_theta=100.0)
    alone = O.attention_prefill(x_q, x_k, x_v, np.arange(n)[None], cfg)[0]
    pad = S - n
    q = np.concatenate([rnd((1, pad, 2, D), 46) * 100, x_q], axis=1)
    k = np.concatenate([rnd((1, pad, 1, D), 47) * 100, x_k], axis=1)
    v = np.concatenate([rnd((1, pad, 1, D), 48) * 100, x_v], axis=1)
    pos = np.concatenate([np.full(pad, 3), np.arange(n)])[None]
    got = O.attention_prefill(q, k, v, pos, cfg, seq_range=np.array([[pad, S]]))[0]
    assert np.max(np.abs(got[pad:] - alone)) < 1e-12
    assert np.all(got[:pad] == 0.0)


def test_right_padding_rows_zero_and_rest_causal():
    S, n, D = 10, 6, 4
    q, k, v = rnd((1, S, 1, D), 49), rnd((1, S, 1, D), 50), rnd((1, S, 1, D), 51)
    pos = np.arange(S)[None]
    cfg = layer(head_dim=D)
    full = O.attention_prefill(q, k, v, pos, cfg)[0]
    got = O.attention_prefill(q, k, v, pos, cfg, seq_range=np.array([[0, n]]))[0]
    assert np.array_equal(got[:n], full[:n])  # causal rows never see keys >= n
    assert np.all(got[n:] == 0.0)


def test_padding_onehot_probe_counts():
    # q = 0: uniform weights over exactly the keys j with max(lo, i-W+1) <= j <= i
    S, D = 9, 9
    qz, kk, v = np.zeros((1, S, 1, D)), rnd((1, S, 1, D), 52), np.eye(S, D)[None, :, None, :]
    for lo in range(0, S):
        for W in (0, 2, 5):
            wts = O.attention_prefill(qz, kk, v, np.arange(S)[None], layer(head_dim=D, window=W),
                                      seq_range=np.array([[lo, S]]))[0, :, 0]
            for i in range(S):
                expect = np.zeros(S)
                if i >= lo:
                    first = lo if W == 0 else max(lo, i - W + 1)
                    expect[first:i + 1] = 1.0 / (i + 1 - first)
                assert np.max(np.abs(wts[i] - expect)) < 1e-15, (lo, W, i)
