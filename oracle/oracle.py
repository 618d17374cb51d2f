"""Float64 CPU oracle for the Gemma 1-4 decoder self-attention forward.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The CUDA library never
calls it and shares no code with it: this file imports numpy and nothing else.

Every step is the plain definition, evaluated in float64 on the (exactly
widened) bf16 input values, in the order the layer applies them:

1. QK-norm (RMSNorm per head over head_dim) -- KerasFormers "Gemma 4", What
   changed (plain-weight RMSNorm, no 1+w offset); Gemma 3's usual 1+w gain;
   norm_eps 1e-6 from the "Gemma" API table; QK-norm itself from the Atlas
   "Gemma 4" summary (RMSNorm pre/post-norm + QK-norm).
2. Rotary embedding, dual bases (KerasFormers "Gemma 3", What changed: rope_theta
   1e6 global / rope_local_theta 1e4 local) with Gemma 4's partial rotation
   (KerasFormers "Gemma 4", What changed: only partial_rotary_factor of each
   head is rotated, the rest passed through).
3. Scaled logits with query_pre_attn_scalar (ZeroModels "Gemma 2", API table).
4. tanh logit softcapping c*tanh(s/c) (ZeroModels "Gemma 2", "Logit
   softcapping" bullet: a scaled tanh).
5. Causal mask, optionally limited to a sliding window (ZeroModels "Gemma 2",
   "Alternating attention" bullet; KerasFormers "Gemma 3" API sliding_window).
6. Softmax over the visible keys and the weighted sum of values; with K=V the
   values are the key tensor as given (KerasFormers "Gemma 4", What changed:
   key and value projections tied).
7. GQA/MQA head grouping: query head h reads kv head h // (H / Hkv)
   (KerasFormers "Gemma" API num_kv_heads=1; ZeroModels "Gemma 2" GQA bullet).
8. An int8 KV cache (Atlas "Gemma 4" summary, long-context/KV section: int8 KV
   caching, Table 3 "+KV"): per-row symmetric codes and an fp32 scale,
   dequantised before step 1 (``kv_quantize``, ``attention_decode_int8``).

Readings taken where the pages are silent:
scale = scalar**-0.5; softcap after scaling; norm before RoPE; V is the raw k
when keys and values are tied; rotated dims are the first R = fraction*D dims,
paired rotate-half (t, t+R/2) with angle pos * theta**(-2t/F), F = head_dim by
default; the window keeps keys with i - j < W; the mask works on token indices
and positions only drive RoPE.

Parity unpinned (no page value fixes them): the frequency denominator F of
partial RoPE, the rotate-half pairing, and the window off-by-one.  The tests
pin the oracle's arithmetic to closed forms, invariants, brute force and a
library routine; they cannot pin those conventions.
"""
from __future__ import annotations

import numpy as np

NORM_NONE = 0
NORM_ONE_PLUS_W = 1
NORM_W = 2


def _f64(x):
    """bf16/fp32 torch tensor or numpy array -> float64 numpy (exact widening)."""
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().float().cpu().numpy()
    return np.asarray(x, dtype=np.float64)


# --- step 1: RMSNorm -------------------------------------------------------

def rms_norm(x, w, mode: int, eps: float):
    """x / sqrt(mean(x^2) + eps) * g over the last axis.

    g = 1 + w (Gemma's usual offset), w (Gemma 4's plain weight), or 1 when
    ``mode`` is NORM_NONE (then this function is the identity and is skipped).
    """
    x = np.asarray(x, dtype=np.float64)
    if mode == NORM_NONE:
        return x
    w = np.asarray(w, dtype=np.float64)
    g = (1.0 + w) if mode == NORM_ONE_PLUS_W else w
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * g


# --- step 2: rotary embedding ----------------------------------------------

def rope_angles(pos, rot_dim: int, theta: float, freq_dim: int):
    """angle[p, t] = pos[p] * theta**(-2t/F) for t < rot_dim/2 (float64)."""
    pos = np.asarray(pos, dtype=np.float64)
    t = np.arange(rot_dim // 2, dtype=np.float64)
    inv_freq = theta ** (-2.0 * t / freq_dim)
    return pos[..., None] * inv_freq


def rope(x, pos, rot_dim: int, theta: float, freq_dim: int):
    """Rotate-half RoPE on dims [0, rot_dim); dims [rot_dim, D) pass through.

    x: [..., D] with pos broadcastable to x.shape[:-1].  For t < R/2, with
    a = x[t], b = x[t+R/2]:  x'[t] = a cos - b sin,  x'[t+R/2] = b cos + a sin.
    """
    x = np.asarray(x, dtype=np.float64)
    if rot_dim == 0:
        return x.copy()
    half = rot_dim // 2
    ang = rope_angles(pos, rot_dim, theta, freq_dim)
    c, s = np.cos(ang), np.sin(ang)
    out = x.copy()
    a = x[..., :half]
    b = x[..., half:rot_dim]
    out[..., :half] = a * c - b * s
    out[..., half:rot_dim] = b * c + a * s
    return out


# --- steps 3-5: logits, softcap, mask ----------------------------------------

def softcap(s, c: float):
    """c * tanh(s / c); c <= 0 means no cap."""
    s = np.asarray(s, dtype=np.float64)
    if c <= 0:
        return s
    return c * np.tanh(s / c)


def visible(i, j, window: int):
    """Key index j is visible to query index i: j <= i and (W == 0 or i - j < W)."""
    i = np.asarray(i)
    j = np.asarray(j)
    ok = j <= i
    if window > 0:
        ok = ok & (i - j < window)
    return ok


def _attend(qt, kt, vals, q_idx, k_idx, scale, cap, window, valid=None):
    """Softmax attention of transformed queries qt [R,D] over keys kt [N,D].

    ``valid`` = (lo, hi) restricts the sequence to token indices [lo, hi): keys
    outside it are masked, and a query outside it (a padding row) sees no key
    and gets a zero output, as does any row with no visible key.
    """
    s = (qt @ kt.T) * scale
    s = softcap(s, cap)
    mask = visible(q_idx[:, None], k_idx[None, :], window)
    if valid is not None:
        lo, hi = valid
        mask = mask & (k_idx[None, :] >= lo) & (q_idx[:, None] >= lo) & (q_idx[:, None] < hi)
    any_vis = mask.any(axis=1)
    s = np.where(mask, s, -np.inf)
    m = np.max(np.where(any_vis[:, None], s, 0.0), axis=1, keepdims=True)
    p = np.where(mask, np.exp(s - m), 0.0)
    den = np.sum(p, axis=1, keepdims=True)
    p = p / np.where(den > 0, den, 1.0)
    return p @ vals


def _layer_fields(cfg):
    get = (lambda k: cfg[k]) if isinstance(cfg, dict) else (lambda k: getattr(cfg, k))
    D = get("head_dim")
    frac = get("rotary_fraction")
    rot = int(round(frac * D))
    fd = get("rope_freq_dim") or D
    return dict(H=get("num_heads"), Hkv=get("num_kv_heads"), D=D, W=get("window"),
                theta=get("rope_theta"), rot=rot, F=fd, cap=get("softcap"),
                scale=float(get("scalar")) ** -0.5, k_eq_v=bool(get("k_eq_v")),
                mode=get("qk_norm"), eps=get("norm_eps"))


# --- the layer: prefill ------------------------------------------------------

def attention_prefill(q, k, v, positions, cfg, w_q=None, w_k=None, rows=None, seq_range=None):
    """Self-attention forward over a whole prompt (float64).

    q [B,S,H,D], k [B,S,Hkv,D], v [B,S,Hkv,D] or None when cfg.k_eq_v,
    positions [B,S] (drive RoPE only).  ``rows`` optionally restricts the
    output to those query indices (same for every b, h).  ``seq_range``
    [B,2] optionally gives each sequence's valid tokens [lo, hi) (a padded
    batch: KerasFormers "Gemma 4", Gemma4Generate.generate argument table,
    `attention_mask` 1 = keep, 0 = padding, and its batched-prompt example); a
    padding token is neither a query nor a key, and padding rows are zero.
    Returns [B,R,H,D].
    """
    f = _layer_fields(cfg)
    q, k, v = _f64(q), _f64(k), _f64(v)
    pos = np.asarray(_f64(positions))
    B, S, H, D = q.shape
    Hkv = k.shape[2]
    assert H == f["H"] and Hkv == f["Hkv"] and D == f["D"] and H % Hkv == 0
    G = H // Hkv
    vals_all = k if f["k_eq_v"] else v
    assert vals_all is not None
    rows = np.arange(S) if rows is None else np.asarray(rows)
    out = np.zeros((B, len(rows), H, D))
    k_idx = np.arange(S)
    for b in range(B):
        kt = rope(rms_norm(k[b], w_k, f["mode"], f["eps"]), pos[b][:, None],
                  f["rot"], f["theta"], f["F"])                      # [S,Hkv,D]
        qt = rope(rms_norm(q[b, rows], w_q, f["mode"], f["eps"]), pos[b, rows][:, None],
                  f["rot"], f["theta"], f["F"])                      # [R,H,D]
        for h in range(H):
            kv = h // G
            valid = None if seq_range is None else (int(seq_range[b][0]), int(seq_range[b][1]))
            out[b, :, h] = _attend(qt[:, h], kt[:, kv], vals_all[b, :, kv], rows, k_idx,
                                   f["scale"], f["cap"], f["W"], valid)
    return out


# --- the layer: one decode step ----------------------------------------------

def attention_decode(q, k_cache, v_cache, seq_lens, cfg, w_q=None, w_k=None, batches=None,
                     first_rows=None, keys_transformed=False):
    """One decode step (float64): query b at position L_b - 1 over cache rows [0, L_b).

    q [B,H,D]; k_cache / v_cache [B,Lmax,Hkv,D] raw (un-normed, un-rotated)
    keys and values, or a list of per-batch [L_b,Hkv,D] arrays; cached key j
    sits at position j.  ``batches`` restricts the output to those batch rows.
    ``first_rows[b]`` (default 0) says the cache given for batch row b starts
    at row first_rows[b]; the rows left out must all be masked, which is
    asserted.  ``keys_transformed``: the cache holds the keys after QK-norm and RoPE
    (k~ of step 2, cached key j rotated at position j), used as they are; only
    for layers whose values are not the keys.  Returns [len(batches),H,D].
    """
    f = _layer_fields(cfg)
    q = _f64(q)
    B, H, D = q.shape
    G = H // f["Hkv"]
    seq_lens = np.asarray(_f64(seq_lens)).astype(np.int64)
    batches = range(B) if batches is None else list(batches)
    out = np.zeros((len(batches), H, D))
    for n, b in enumerate(batches):
        L = int(seq_lens[b])
        r0 = 0 if first_rows is None else int(first_rows[b])
        assert r0 == 0 or not visible(L - 1, r0 - 1, f["W"]), "a visible cache row was left out"
        kc = _f64(k_cache[b])[:L - r0]
        vc = kc if f["k_eq_v"] else _f64(v_cache[b])[:L - r0]
        pos_k = np.arange(r0, L)
        if keys_transformed:
            assert not f["k_eq_v"], "tied values need the raw keys"
            kt = kc
        else:
            kt = rope(rms_norm(kc, w_k, f["mode"], f["eps"]), pos_k[:, None],
                      f["rot"], f["theta"], f["F"])
        qt = rope(rms_norm(q[b], w_q, f["mode"], f["eps"]), np.array([L - 1]),
                  f["rot"], f["theta"], f["F"])                       # [H,D]
        for h in range(H):
            kv = h // G
            out[n, h] = _attend(qt[h:h + 1], kt[:, kv], vc[:, kv], np.array([L - 1]), pos_k,
                                f["scale"], f["cap"], f["W"])[0]
    return out


def attention_prefill_chunk(q, k_cache, v_cache, prefix_lens, cfg, w_q=None, w_k=None, rows=None,
                            keys_transformed=False):
    """A chunk of C new tokens against a cached prefix (float64): the prompt in pieces.

    KerasFormers "Gemma 4", Gemma4Generate.generate runs the model over a prompt
    and then token by token with a cache; a chunk is the general step between the
    two.  Sequence b holds P_b = prefix_lens[b] cached tokens; the chunk's C
    tokens sit at positions P_b .. P_b + C - 1, and their keys/values are already
    in the cache at rows P_b .. P_b + C - 1.  Query i attends to cache rows
    [0, P_b + i] (within the window), cached key j at position j (raw keys and
    values, as attention_decode takes them).
    q [B,C,H,D]; k_cache / v_cache [B,Lmax,Hkv,D] (v_cache None when k_eq_v).
    ``rows`` optionally restricts the output to those chunk rows;
    ``keys_transformed`` as in attention_decode.  Returns [B,R,H,D].
    """
    f = _layer_fields(cfg)
    q = _f64(q)
    B, C, H, D = q.shape
    G = H // f["Hkv"]
    prefix_lens = np.asarray(_f64(prefix_lens)).astype(np.int64)
    rows = np.arange(C) if rows is None else np.asarray(rows)
    out = np.zeros((B, len(rows), H, D))
    for b in range(B):
        P = int(prefix_lens[b])
        n = P + C                                   # cache rows the chunk can see
        kc = _f64(k_cache[b])[:n]
        vc = kc if f["k_eq_v"] else _f64(v_cache[b])[:n]
        k_idx = np.arange(n)                        # cached key j: token j, position j
        q_idx = P + rows                            # chunk token i: token P + i
        if keys_transformed:
            assert not f["k_eq_v"], "tied values need the raw keys"
            kt = kc
        else:
            kt = rope(rms_norm(kc, w_k, f["mode"], f["eps"]), k_idx[:, None], f["rot"], f["theta"], f["F"])
        qt = rope(rms_norm(q[b, rows], w_q, f["mode"], f["eps"]), q_idx[:, None], f["rot"], f["theta"], f["F"])
        for h in range(H):
            kv = h // G
            out[b, :, h] = _attend(qt[:, h], kt[:, kv], vc[:, kv], q_idx, k_idx, f["scale"], f["cap"], f["W"])
    return out


def transform_keys(k_rows, positions, cfg, w_k=None):
    """The keys a transformed cache holds: RoPE(QK-norm(k)) of rows k_rows [N,Hkv,D] at
    ``positions`` [N] (steps 1-2), float64."""
    f = _layer_fields(cfg)
    return rope(rms_norm(_f64(k_rows), w_k, f["mode"], f["eps"]), np.asarray(positions)[:, None],
                f["rot"], f["theta"], f["F"])


# --- split-KV merge (decode's two-stage form) ---------------------------------

def lse_merge(parts):
    """Merge per-chunk softmax partials (m, l, O) of one query row.

    Each chunk c contributes m_c = max of its logits, l_c = sum exp(s - m_c),
    O_c = sum exp(s - m_c) v.  The merged row is
    sum_c e^(m_c - M) O_c / sum_c e^(m_c - M) l_c with M = max_c m_c.
    """
    M = max(m for m, _, _ in parts)
    num = sum(np.exp(m - M) * o for m, _, o in parts)
    den = sum(np.exp(m - M) * l for m, l, _ in parts)
    return num / den


def chunk_partial(s, vals):
    """(m, l, O) of one chunk: logits s [n] (already capped and masked), values [n,D]."""
    m = np.max(s)
    p = np.exp(s - m)
    return m, np.sum(p), p @ vals


# --- int8 KV cache ---------------------------------------------------------------

def kv_quantize(x):
    """Symmetric int8 codes of cache rows, one fp32 scale per row (float32 arithmetic).

    The Atlas summary of the Gemma 4 report lists int8 KV caching (Table 3, "+KV")
    without its format; the reading here: each row x (the head_dim values of one
    position and kv head) gets scale s = max|x| / 127 and codes
    c = round-half-even(x / s) clipped to [-127, 127], so that c * s is the
    dequantised row.  Both divisions are IEEE float32 (correctly rounded): the
    codes are integers decided by floating point, so the precision is fixed here.
    A row of zeros gets s = 0 and codes 0.  x [..., D] -> (int8 [..., D], fp32 [...]).
    """
    x = np.asarray(_f64(x), dtype=np.float32)
    amax = np.max(np.abs(x), axis=-1)
    s = (amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    c = np.rint((x / safe[..., None]).astype(np.float32))
    c = np.clip(c, -127, 127)
    c = np.where((s > 0)[..., None], c, 0.0)
    return c.astype(np.int8), s


def kv_dequantize(codes, scales):
    """codes [..., D] int8 times their row's scale [...], in float64."""
    return np.asarray(codes, dtype=np.float64) * np.asarray(scales, dtype=np.float64)[..., None]


def attention_decode_int8(q, k_codes, k_scales, v_codes, v_scales, seq_lens, cfg, w_q=None, w_k=None,
                          batches=None, first_rows=None, keys_transformed=False):
    """One decode step over an int8 cache: attention_decode on the dequantised rows.

    k_codes / v_codes [B,Lmax,Hkv,D] int8 (or per-batch lists, as attention_decode
    takes), k_scales / v_scales [B,Lmax,Hkv] (or lists); with K=V the values are
    the dequantised raw keys (v_codes / v_scales unused).
    """
    f = _layer_fields(cfg)

    def deq(codes, scales):  # batch rows given as None are left out (see ``batches``)
        return [None if codes[b] is None else kv_dequantize(codes[b], scales[b]) for b in range(len(codes))]

    kd = deq(k_codes, k_scales)
    vd = None if f["k_eq_v"] else deq(v_codes, v_scales)
    return attention_decode(q, kd, vd, seq_lens, cfg, w_q=w_q, w_k=w_k, batches=batches,
                            first_rows=first_rows, keys_transformed=keys_transformed)
