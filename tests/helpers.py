"""Shared test plumbing: device copies of seeded inputs and error statistics."""
import numpy as np
import torch

import workloads as W

MAX_ABS = 2e-2   # bf16 inputs, fp32 accumulation, bf16 output
MEAN_ABS = 2e-3


def err_stats(got, ref):
    g = got.detach().float().cpu().numpy().astype(np.float64) if hasattr(got, "detach") else got
    d = np.abs(g - ref)
    return float(d.max()), float(d.mean())


def assert_close(got, ref, what=""):
    mx, mean = err_stats(got, ref)
    assert np.isfinite(mx), f"{what}: non-finite output"
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max-abs {mx:.3e} mean-abs {mean:.3e}"
    return mx, mean


def make_layer(layer: W.Layer, max_pos: int, w_q=None, w_k=None):
    from gemma_family_decoder_b200 import AttentionLayer, LayerSpec
    return AttentionLayer(LayerSpec.of(layer), max_pos, w_q, w_k)


def to_dev(d: dict, keys=("q", "k", "v", "positions")):
    return {k: (None if d.get(k) is None else d[k].cuda().contiguous()) for k in keys}


def small_prefill_inputs(layer: W.Layer, B: int, S: int, seed: int, gain_mean=0.0):
    wl = W.PrefillWorkload("t", layer, B, S, seed, gain_mean=gain_mean)
    return W.prefill_inputs(wl)


def decode_full_cache(wl: W.DecodeWorkload, seq_lens, max_len=None, layer=None, device="cuda"):
    """Device caches [B,Lmax,Hkv,D] holding the rows each query can see, plus host copies.

    Rows a query never sees stay NaN on the device, so a kernel that reads them
    shows up in its output.  Returns (k_dev, v_dev, oracle_args) where
    oracle_args = dict(k_cache=[rows], v_cache=[rows] or None, first_rows=[...])
    holds only the visible rows of each batch row for the oracle.
    """
    layer = layer or wl.layer
    B = len(seq_lens)
    Lmax = max_len or wl.max_len
    shape = (B, Lmax, layer.num_kv_heads, layer.head_dim)
    k = torch.full(shape, float("nan"), dtype=torch.bfloat16, device=device)
    v = None if layer.k_eq_v else torch.full(shape, float("nan"), dtype=torch.bfloat16, device=device)
    ks, vs, firsts = [], [], []
    for b in range(B):
        L = int(seq_lens[b])
        lo = 0 if layer.window == 0 else max(0, L - layer.window)
        rows = W.decode_cache_rows(wl, b, L - lo, lo, layer=layer)
        k[b, lo:L] = rows["k"].to(device)
        ks.append(rows["k"])
        if v is not None:
            v[b, lo:L] = rows["v"].to(device)
            vs.append(rows["v"])
        firsts.append(lo)
    return k, v, dict(k_cache=ks, v_cache=vs if v is not None else None, first_rows=firsts)
