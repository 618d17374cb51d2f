"""GPU parity of caches holding transformed keys (gattn_cfg.keys_transformed).

The library writes the keys QK-normed and rotated at their positions
(gattn_kv_append_layer, gattn_prefill_chunk's append); the decode kernels (CUDA-core,
fallback split, int8) and the chunk prefill then read them as they are.  Checked
against the oracle with ``keys_transformed`` on the cache the library wrote, and
against the raw-cache results; the written keys against ``transform_keys``.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from helpers import assert_close, decode_full_cache, make_layer, small_prefill_inputs

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def tk_layer(layer, max_pos, w_q=None, w_k=None):
    from gemma_family_decoder_b200 import AttentionLayer, LayerSpec
    spec = dataclasses.replace(LayerSpec.of(layer), keys_transformed=True)
    return AttentionLayer(spec, max_pos, w_q, w_k)


def transformed_cache(L, wl, layer, seq_lens, Lmax):
    """Raw visible rows appended through the library into zeroed caches; returns the
    transformed device caches, the raw oracle rows and the first visible rows."""
    k, v, oa = decode_full_cache(wl, seq_lens, max_len=Lmax, layer=layer)
    kc = torch.zeros_like(k)
    vc = torch.zeros_like(v)
    for b in range(len(seq_lens)):
        lo, n = oa["first_rows"][b], int(seq_lens[b])
        L.kv_append(oa["k_cache"][b][None].cuda().contiguous(), oa["v_cache"][b][None].cuda().contiguous(),
                    kc[b:b + 1], vc[b:b + 1], torch.tensor([lo], dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    return kc, vc, oa


CASES = [
    ("local_g2_w1024", W.GEMMA4_DECODE_LOCAL.layer, [1, 300, 1025, 2000]),
    ("g4_norm_partial", W.Layer(num_heads=8, num_kv_heads=2, head_dim=256, rotary_fraction=0.25,
                                qk_norm=W.NORM_W), [5, 700]),
    ("g1_d512_norm1_cap", W.Layer(num_heads=2, num_kv_heads=2, head_dim=512, scalar=512.0, softcap=30.0,
                                  qk_norm=W.NORM_ONE_PLUS_W, window=300), [9, 301, 640]),
    ("fallback_g8", W.Layer(num_heads=16, num_kv_heads=2, head_dim=256, rope_theta=1e6), [3, 513]),
]


@pytest.mark.parametrize("name,layer,lens", CASES, ids=[c[0] for c in CASES])
def test_decode_over_transformed_cache(name, layer, lens):
    gm = 1.0 if layer.qk_norm == W.NORM_W else 0.0
    wl = W.DecodeWorkload(name, layer, len(lens), 1, max(lens), seed=31, gain_mean=gm)
    dq = W.decode_inputs(wl, layer=layer)
    seq_lens = torch.tensor(lens, dtype=torch.int32)
    Lmax = max(lens) + 3
    L = tk_layer(layer, Lmax, dq["w_q"], dq["w_k"])
    kc, vc, oa = transformed_cache(L, wl, layer, seq_lens, Lmax)
    # the written keys are the transformed rows, to bf16 rounding
    for b, lo in enumerate(oa["first_rows"]):
        n = int(seq_lens[b])
        ref = O.transform_keys(oa["k_cache"][b], np.arange(lo, n), layer, w_k=dq["w_k"])
        got = kc[b, lo:n].double().cpu().numpy()
        assert np.max(np.abs(got - ref)) <= 2e-2 * max(1.0, np.max(np.abs(ref)))
    out = L.decode(dq["q"].cuda(), kc, vc, seq_lens.cuda())
    torch.cuda.synchronize()
    kt_rows = [kc[b, lo:int(seq_lens[b])].cpu() for b, lo in enumerate(oa["first_rows"])]
    ref = O.attention_decode(dq["q"], kt_rows, oa["v_cache"], seq_lens, layer, w_q=dq["w_q"], w_k=dq["w_k"],
                             first_rows=oa["first_rows"], keys_transformed=True)
    assert_close(out, ref, name)
    raw = O.attention_decode(dq["q"], oa["k_cache"], oa["v_cache"], seq_lens, layer, w_q=dq["w_q"], w_k=dq["w_k"],
                             first_rows=oa["first_rows"])
    assert_close(out, raw, name + " vs raw keys")


def test_int8_over_transformed_cache():
    layer = W.GEMMA4_DECODE_LOCAL.layer
    lens = [64, 1024, 1500]
    wl = W.DecodeWorkload("i8tk", layer, 3, 1, max(lens), seed=33)
    dq = W.decode_inputs(wl, layer=layer)
    seq_lens = torch.tensor(lens, dtype=torch.int32)
    Lmax = max(lens)
    L = tk_layer(layer, Lmax)
    kc, vc, oa = transformed_cache(L, wl, layer, seq_lens, Lmax)
    from gemma_family_decoder_b200 import kv_quantize
    kq, ks = kv_quantize(kc)
    vq, vs = kv_quantize(vc)
    out = L.decode_int8(dq["q"].cuda(), kq, ks, vq, vs, seq_lens.cuda())
    torch.cuda.synchronize()
    kcs, kss, vcs, vss = [], [], [], []
    for b, lo in enumerate(oa["first_rows"]):
        n = int(seq_lens[b])
        c, s = O.kv_quantize(kc[b, lo:n].float().cpu().numpy())
        assert np.array_equal(kq[b, lo:n].cpu().numpy(), c)
        kcs.append(c)
        kss.append(s)
        c, s = O.kv_quantize(oa["v_cache"][b].float().numpy())
        vcs.append(c)
        vss.append(s)
    ref = O.attention_decode_int8(dq["q"], kcs, kss, vcs, vss, seq_lens, layer, first_rows=oa["first_rows"],
                                  keys_transformed=True)
    assert_close(out, ref, "int8 over transformed keys")


@pytest.mark.parametrize("over", [dict(), dict(qk_norm=W.NORM_W, window=100, softcap=40.0)])
def test_chunks_over_transformed_cache_equal_whole_prompt(over):
    layer = W.Layer(**{**dict(num_heads=4, num_kv_heads=2, head_dim=256, scalar=256.0), **over})
    sizes = [130, 1, 97]
    S = sum(sizes)
    gm = 1.0 if layer.qk_norm == W.NORM_W else 0.0
    d = small_prefill_inputs(layer, 2, S, seed=35, gain_mean=gm)
    Lraw = make_layer(layer, S, d["w_q"], d["w_k"])
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    whole = Lraw.prefill(q, k, v, d["positions"].cuda())
    L = tk_layer(layer, S, d["w_q"], d["w_k"])
    kc = torch.zeros_like(k)
    vc = torch.zeros_like(v)
    outs, p = [], 0
    for n in sizes:
        pre = torch.full((2,), p, dtype=torch.int32, device="cuda")
        sl = slice(p, p + n)
        outs.append(L.prefill_chunk(q[:, sl].contiguous(), kc, vc, pre, k_new=k[:, sl].contiguous(),
                                    v_new=v[:, sl].contiguous()))
        p += n
    torch.cuda.synchronize()
    assert torch.equal(vc, v)
    for b in range(2):
        ref = O.transform_keys(d["k"][b], np.arange(S), layer, w_k=d["w_k"])
        assert np.max(np.abs(kc[b].double().cpu().numpy() - ref)) <= 2e-2 * max(1.0, np.max(np.abs(ref)))
    assert_close(torch.cat(outs, dim=1), whole.double().cpu().numpy(), "chunks over transformed keys")
    ref = O.attention_prefill_chunk(d["q"][:, S - sizes[-1]:], kc.cpu(), vc.cpu(), [S - sizes[-1]] * 2, layer,
                                    w_q=d["w_q"], w_k=d["w_k"], keys_transformed=True)
    assert_close(outs[-1], ref, "last chunk vs oracle")


def test_transformed_flag_refused_with_tied_values():
    from gemma_family_decoder_b200 import GattnError
    layer = W.Layer(num_heads=4, num_kv_heads=1, head_dim=512, scalar=512.0, k_eq_v=True, rotary_fraction=0.25)
    L = tk_layer(layer, 64)
    q = torch.zeros(1, 4, 512, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(1, 64, 1, 512, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(GattnError):
        L.decode(q, kc, None, torch.tensor([5], dtype=torch.int32, device="cuda"))
