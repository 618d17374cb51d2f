"""Seeded synthetic inputs for the Gemma self-attention layer workloads.

This module only describes workload shapes and draws random numbers.  It holds
none of the attention arithmetic: both the float64 oracle (``oracle/``) and the
CUDA library (``gemma_family_decoder_b200``) consume what it produces, and it
imports neither of them.

Draw recipe (every tensor comes from a CPU ``torch.Generator`` seeded per
workload, fp32 ``randn`` rounded to bf16):

* prefill: ``q`` [B,S,H,D], then ``k`` [B,S,Hkv,D], then ``v`` (omitted when the
  layer ties keys and values), then the QK-norm gains ``w_q``, ``w_k`` [D]
  (fp32) when the layer has QK-norm.  Positions are ``0..S-1`` per sequence.
* decode: ``seq_lens`` [B] uniform in ``[lo, hi]`` from the workload seed, then
  ``q`` [B,H,D]; each batch row's cache rows are drawn from their own generator
  seeded ``(seed, b)`` so that a single row can be regenerated on its own.

The layer parameters follow the model cards' argument tables: KerasFormers
"Gemma" (API: num_heads 8, num_kv_heads 1, head_dim 256, rope_theta 1e4),
ZeroModels "Gemma 2" (API: query_pre_attn_scalar 256, attn_logit_softcapping 50,
num_kv_heads 4), KerasFormers "Gemma 3" (API: sliding_window 512, rope_theta 1e6
global / 1e4 local, norm_eps 1e-6) and KerasFormers "Gemma 4" (What changed;
API: num_global_kv_heads 1, global_head_dim 512, k_eq_v, sliding_window 1024,
partial_rotary_factor 0.25).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import torch

NORM_NONE = 0
NORM_ONE_PLUS_W = 1  # Gemma 3 style gain (1 + w)
NORM_W = 2           # Gemma 4 style plain gain w


@dataclasses.dataclass(frozen=True)
class Layer:
    """Attention-layer parameters (the fields of the library's ``gattn_cfg``)."""

    num_heads: int
    num_kv_heads: int
    head_dim: int
    window: int = 0               # 0 = full causal
    rope_theta: float = 10000.0
    rotary_fraction: float = 1.0  # fraction of each head that is rotated
    rope_freq_dim: int = 0        # F in theta^(-2t/F); 0 means head_dim
    softcap: float = 0.0          # 0 = off
    scalar: float = 256.0         # query_pre_attn_scalar; scale = scalar^-1/2
    k_eq_v: bool = False
    qk_norm: int = NORM_NONE
    norm_eps: float = 1e-6

    @property
    def rot_dim(self) -> int:
        return int(round(self.rotary_fraction * self.head_dim))

    @property
    def freq_dim(self) -> int:
        return self.rope_freq_dim or self.head_dim


@dataclasses.dataclass(frozen=True)
class PrefillWorkload:
    name: str
    layer: Layer
    batch: int
    seq: int
    seed: int
    gain_mean: float = 0.0   # w ~ gain_mean + N(0, gain_std)
    gain_std: float = 0.1
    # > 0: a left-padded batch of prompts (KerasFormers "Gemma 4", Gemma4Generate.generate,
    # attention_mask), sequence b holding the last n_b tokens, n_b ~ U[len_lo, seq]
    len_lo: int = 0


@dataclasses.dataclass(frozen=True)
class ChunkWorkload:
    """The last ``chunk`` tokens of a ``prefix + chunk`` prompt, the first ``prefix``
    already in the cache (KerasFormers "Gemma 4", Gemma4Generate.generate, in pieces)."""
    name: str
    layer: Layer
    batch: int
    prefix: int
    chunk: int
    seed: int
    gain_mean: float = 0.0
    gain_std: float = 0.1
    keys_transformed: bool = False   # the cache holds transformed keys


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    layer: Layer
    batch: int
    len_lo: int
    len_hi: int
    seed: int
    gain_mean: float = 0.0
    gain_std: float = 0.1
    # the cache held as int8 codes + fp32 row scales (Atlas "Gemma 4" summary: int8 KV
    # caching), quantised from the same bf16 rows
    kv_int8: bool = False
    # the cache holds the keys after QK-norm and RoPE (written by the library's append)
    keys_transformed: bool = False

    @property
    def max_len(self) -> int:
        return self.len_hi


# --- the five workloads ------------------------------------------------------

GEMMA2_LOCAL = PrefillWorkload(
    "gemma2_2b_local_s256",
    Layer(num_heads=8, num_kv_heads=4, head_dim=256, window=128, rope_theta=1e4,
          softcap=50.0, scalar=256.0),
    batch=1, seq=256, seed=0)

GEMMA1_MQA = PrefillWorkload(
    "gemma1_2b_mqa_b4_s2048",
    Layer(num_heads=8, num_kv_heads=1, head_dim=256, window=0, rope_theta=1e4,
          scalar=256.0),
    batch=4, seq=2048, seed=1)

_G3 = dict(num_heads=4, num_kv_heads=1, head_dim=256, scalar=256.0,
           qk_norm=NORM_ONE_PLUS_W, norm_eps=1e-6)
GEMMA3_LOCAL = PrefillWorkload(
    "gemma3_1b_local_w512_b2_s8192",
    Layer(window=512, rope_theta=1e4, **_G3), batch=2, seq=8192, seed=2)
GEMMA3_GLOBAL = PrefillWorkload(
    "gemma3_1b_global_b2_s8192",
    Layer(window=0, rope_theta=1e6, **_G3), batch=2, seq=8192, seed=2)
# the 5:1 pattern: five local layers then one global layer, same inputs
GEMMA3_PATTERN: List[PrefillWorkload] = [GEMMA3_LOCAL] * 5 + [GEMMA3_GLOBAL]

GEMMA4_GLOBAL = PrefillWorkload(
    "gemma4_12b_global_keqv_s32768",
    Layer(num_heads=16, num_kv_heads=1, head_dim=512, window=0, rope_theta=1e6,
          rotary_fraction=0.25, scalar=512.0, k_eq_v=True, qk_norm=NORM_W,
          norm_eps=1e-6),
    batch=1, seq=32768, seed=3, gain_mean=1.0, gain_std=0.1)

GEMMA4_DECODE_LOCAL = DecodeWorkload(
    "gemma4_12b_decode_local_b64",
    Layer(num_heads=16, num_kv_heads=8, head_dim=256, window=1024,
          rope_theta=1e4, scalar=256.0),
    batch=64, len_lo=1024, len_hi=32768, seed=4)
GEMMA4_DECODE_GLOBAL = DecodeWorkload(
    "gemma4_12b_decode_global_keqv_b64",
    Layer(num_heads=16, num_kv_heads=1, head_dim=512, window=0, rope_theta=1e6,
          rotary_fraction=0.25, scalar=512.0, k_eq_v=True),
    batch=64, len_lo=1024, len_hi=32768, seed=4)
# an added decode row exercising the Gemma 4 plain-w QK-norm in the K prologue
GEMMA4_DECODE_GLOBAL_NORM = DecodeWorkload(
    "gemma4_12b_decode_global_keqv_qknorm_b64",
    dataclasses.replace(GEMMA4_DECODE_GLOBAL.layer, qk_norm=NORM_W),
    batch=64, len_lo=1024, len_hi=32768, seed=4, gain_mean=1.0, gain_std=0.1)

# a batch of eight prompts of 512 to 4096 tokens, left-padded to 4096, through the
# Gemma 3 global layer
GEMMA3_GLOBAL_LEFTPAD = PrefillWorkload(
    "gemma3_1b_global_b8_s4096_leftpad",
    Layer(window=0, rope_theta=1e6, **_G3), batch=8, seq=4096, seed=5, len_lo=512)

# the local decode layer over an int8 cache of the same rows
GEMMA4_DECODE_LOCAL_INT8 = dataclasses.replace(GEMMA4_DECODE_LOCAL, name="gemma4_12b_decode_local_int8_b64",
                                               kv_int8=True)

# the last 1024-token chunk of eight 8192-token prompts through the Gemma 3 global layer
GEMMA3_GLOBAL_CHUNK = ChunkWorkload(
    "gemma3_1b_global_b8_chunk1024_prefix7168",
    Layer(window=0, rope_theta=1e6, **_G3), batch=8, prefix=7168, chunk=1024, seed=6)

# the global K=V decode over an int8 cache (the tensor-core decode, on the codes)
GEMMA4_DECODE_GLOBAL_INT8 = dataclasses.replace(GEMMA4_DECODE_GLOBAL, name="gemma4_12b_decode_global_keqv_int8_b64",
                                                kv_int8=True)
# the same decode and chunk steps over caches holding transformed keys
GEMMA4_DECODE_LOCAL_TK = dataclasses.replace(GEMMA4_DECODE_LOCAL, name="gemma4_12b_decode_local_tk_b64",
                                             keys_transformed=True)
GEMMA4_DECODE_LOCAL_INT8_TK = dataclasses.replace(GEMMA4_DECODE_LOCAL, name="gemma4_12b_decode_local_int8_tk_b64",
                                                  kv_int8=True, keys_transformed=True)
GEMMA3_GLOBAL_CHUNK_TK = dataclasses.replace(GEMMA3_GLOBAL_CHUNK, name="gemma3_1b_global_b8_chunk1024_prefix7168_tk",
                                             keys_transformed=True)

PREFILL: Dict[str, PrefillWorkload] = {w.name: w for w in (
    GEMMA2_LOCAL, GEMMA1_MQA, GEMMA3_LOCAL, GEMMA3_GLOBAL, GEMMA4_GLOBAL, GEMMA3_GLOBAL_LEFTPAD)}
DECODE: Dict[str, DecodeWorkload] = {w.name: w for w in (
    GEMMA4_DECODE_LOCAL, GEMMA4_DECODE_GLOBAL, GEMMA4_DECODE_GLOBAL_NORM, GEMMA4_DECODE_LOCAL_INT8,
    GEMMA4_DECODE_LOCAL_TK, GEMMA4_DECODE_LOCAL_INT8_TK, GEMMA4_DECODE_GLOBAL_INT8)}


# --- drawing -------------------------------------------------------------------

def _randn_bf16(gen: torch.Generator, shape) -> torch.Tensor:
    return torch.randn(shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)


def _gains(gen: torch.Generator, layer: Layer, mean: float, std: float):
    if layer.qk_norm == NORM_NONE:
        return None, None
    D = layer.head_dim
    w_q = mean + std * torch.randn(D, generator=gen, dtype=torch.float32)
    w_k = mean + std * torch.randn(D, generator=gen, dtype=torch.float32)
    return w_q, w_k


def prefill_inputs(wl: PrefillWorkload, batch: Optional[int] = None,
                   seq: Optional[int] = None, layer: Optional[Layer] = None) -> dict:
    """Draw q, k, v, positions and gains for a prefill workload.

    ``batch``/``seq``/``layer`` override the workload's own values (smaller
    cases for tests); the draw order stays the same.
    """
    layer = layer or wl.layer
    B = batch or wl.batch
    S = seq or wl.seq
    H, Hkv, D = layer.num_heads, layer.num_kv_heads, layer.head_dim
    gen = torch.Generator().manual_seed(wl.seed)
    q = _randn_bf16(gen, (B, S, H, D))
    k = _randn_bf16(gen, (B, S, Hkv, D))
    v = None if layer.k_eq_v else _randn_bf16(gen, (B, S, Hkv, D))
    w_q, w_k = _gains(gen, layer, wl.gain_mean, wl.gain_std)
    positions = torch.arange(S, dtype=torch.int32).unsqueeze(0).repeat(B, 1)
    seq_range = None
    if wl.len_lo > 0:
        # left padding: sequence b keeps tokens [S - n_b, S), numbered 0, 1, ... from the
        # first kept one; padding tokens sit at position 0 (a shorter S scales len_lo)
        n_lo = max(1, wl.len_lo * S // wl.seq)
        n = torch.randint(n_lo, S + 1, (B,), generator=gen, dtype=torch.int64)
        lo = (S - n).to(torch.int32)
        seq_range = torch.stack([lo, torch.full_like(lo, S)], dim=1).contiguous()
        t = torch.arange(S, dtype=torch.int32).unsqueeze(0)
        positions = torch.clamp(t - lo.unsqueeze(1), min=0).to(torch.int32).contiguous()
    return dict(q=q, k=k, v=v, positions=positions, w_q=w_q, w_k=w_k, layer=layer,
                seq_range=seq_range)


def chunk_inputs(wl: ChunkWorkload) -> dict:
    """The whole prompt drawn as a prefill of prefix + chunk tokens (same draw order),
    split into the cache (rows [0, prefix), zeros past them) and the chunk's q, k, v."""
    n = wl.prefix + wl.chunk
    d = prefill_inputs(PrefillWorkload(wl.name, wl.layer, wl.batch, n, wl.seed, wl.gain_mean, wl.gain_std))
    P, C = wl.prefix, wl.chunk
    k_cache = torch.zeros_like(d["k"])
    k_cache[:, :P] = d["k"][:, :P]
    v_cache = None
    if d["v"] is not None:
        v_cache = torch.zeros_like(d["v"])
        v_cache[:, :P] = d["v"][:, :P]
    return dict(q=d["q"][:, P:].contiguous(), k_new=d["k"][:, P:].contiguous(),
                v_new=None if d["v"] is None else d["v"][:, P:].contiguous(), k_cache=k_cache, v_cache=v_cache,
                prefix_lens=torch.full((wl.batch,), P, dtype=torch.int32), w_q=d["w_q"], w_k=d["w_k"],
                layer=wl.layer, max_len=n)


def decode_inputs(wl: DecodeWorkload, batch: Optional[int] = None,
                  len_lo: Optional[int] = None, len_hi: Optional[int] = None,
                  layer: Optional[Layer] = None) -> dict:
    """Draw ``seq_lens`` [B] int32, then the query [B,H,D], then the gains.

    ``seq_lens[b]`` counts the current token: its query sits at position
    ``seq_lens[b]-1`` and cache rows ``0..seq_lens[b]-1`` hold its keys.
    """
    layer = layer or wl.layer
    B = batch or wl.batch
    lo = len_lo or wl.len_lo
    hi = len_hi or wl.len_hi
    gen = torch.Generator().manual_seed(wl.seed)
    seq_lens = torch.randint(lo, hi + 1, (B,), generator=gen, dtype=torch.int64).to(torch.int32)
    q = _randn_bf16(gen, (B, layer.num_heads, layer.head_dim))
    w_q, w_k = _gains(gen, layer, wl.gain_mean, wl.gain_std)
    return dict(seq_lens=seq_lens, q=q, w_q=w_q, w_k=w_k, layer=layer)


def decode_cache_rows(wl: DecodeWorkload, b: int, rows: int, start: int = 0,
                      layer: Optional[Layer] = None) -> dict:
    """Cache rows ``[start, start+rows)`` of batch row ``b``: k (and v) [rows,Hkv,D].

    Each batch row has its own generator per 1024-row block, seeded from
    ``(seed, b, block)``, so any range of rows can be regenerated on its own.
    """
    layer = layer or wl.layer
    Hkv, D = layer.num_kv_heads, layer.head_dim
    blk = 1024
    if rows <= 0:
        e = torch.empty(0, Hkv, D, dtype=torch.bfloat16)
        return dict(k=e, v=None if layer.k_eq_v else e.clone())
    first, last = start // blk, (start + rows - 1) // blk
    ks, vs = [], []
    for blk_i in range(first, last + 1):
        gen = torch.Generator().manual_seed(wl.seed * 1_000_003 + b * 65_537 + blk_i)
        ks.append(_randn_bf16(gen, (blk, Hkv, D)))
        if not layer.k_eq_v:
            vs.append(_randn_bf16(gen, (blk, Hkv, D)))
    off = start - first * blk
    k = torch.cat(ks)[off:off + rows]
    v = None if layer.k_eq_v else torch.cat(vs)[off:off + rows]
    return dict(k=k, v=v)
