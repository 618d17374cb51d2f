"""GPU parity of chunked prefill against a cached prefix (gattn_prefill_chunk) and the
cache append (gattn_kv_append), against the oracle's ``attention_prefill_chunk``.

Caches start as zeros past each sequence's prefix (cache rows past the chunk are
read with weight 0 by the last key tile and must be finite); the chunk's own rows
arrive through the library's append.  Tolerance: max-abs 2e-2, mean-abs 2e-3.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from helpers import assert_close, make_layer, small_prefill_inputs, to_dev

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def chunk_case(layer, prefixes, C, pad, seed):
    """Full per-sequence token draws of length max(prefix) + C + pad, the prefix rows
    in the cache (zeros past them), and the chunk's q, k, v."""
    B = len(prefixes)
    Lmax = max(prefixes) + C + pad
    gm = 1.0 if layer.qk_norm == W.NORM_W else 0.0
    d = small_prefill_inputs(layer, B, Lmax, seed=seed, gain_mean=gm)
    k_cache = torch.zeros_like(d["k"])
    v_cache = None if layer.k_eq_v else torch.zeros_like(d["v"])
    q = torch.stack([d["q"][b, p:p + C] for b, p in enumerate(prefixes)])
    k_new = torch.stack([d["k"][b, p:p + C] for b, p in enumerate(prefixes)])
    v_new = None if layer.k_eq_v else torch.stack([d["v"][b, p:p + C] for b, p in enumerate(prefixes)])
    for b, p in enumerate(prefixes):
        k_cache[b, :p] = d["k"][b, :p]
        if v_cache is not None:
            v_cache[b, :p] = d["v"][b, :p]
    return d, dict(q=q, k_new=k_new, v_new=v_new, k_cache=k_cache, v_cache=v_cache, Lmax=Lmax)


def run_chunk(layer, d, c, prefixes, append=True):
    L = make_layer(layer, c["Lmax"], d["w_q"], d["w_k"])
    dev = {k: (None if c[k] is None else c[k].cuda().contiguous()) for k in ("q", "k_new", "v_new", "k_cache",
                                                                             "v_cache")}
    pre = torch.tensor(prefixes, dtype=torch.int32, device="cuda")
    ws = L.prefill_chunk_workspace(len(prefixes), c["q"].shape[1], c["Lmax"])
    if not append:  # the chunk's rows are already in the cache
        from gemma_family_decoder_b200 import kv_append
        kv_append(dev["k_new"], dev["v_new"], dev["k_cache"], dev["v_cache"], pre, status=ws)
    out = L.prefill_chunk(dev["q"], dev["k_cache"], dev["v_cache"], pre,
                          k_new=dev["k_new"] if append else None, v_new=dev["v_new"] if append else None,
                          workspace=ws)
    from gemma_family_decoder_b200 import check
    st = check(ws)
    return out, st, dev


BASE = dict(num_heads=4, num_kv_heads=2, head_dim=256, scalar=256.0)
CASES = [
    # (name, layer overrides, per-sequence prefixes, C)
    ("gqa_c130", dict(), [0, 5, 200], 130),
    ("gqa_c1", dict(), [0, 77, 300], 1),
    ("mqa_c17_norope", dict(num_heads=8, num_kv_heads=1, rotary_fraction=0.0), [3, 128, 129], 17),
    ("window7_c257", dict(window=7), [0, 40, 130], 257),
    ("window128_softcap_c200", dict(window=128, softcap=50.0), [100, 255, 0], 200),
    ("qknorm1_c64", dict(qk_norm=W.NORM_ONE_PLUS_W, rope_theta=1e6), [1, 63, 64], 64),
    ("keqv_d512_norm_partial", dict(head_dim=512, num_heads=4, num_kv_heads=1, k_eq_v=True, rotary_fraction=0.25,
                                    rope_theta=1e6, qk_norm=W.NORM_W, scalar=512.0), [0, 70, 190], 129),
    ("d512_window100", dict(head_dim=512, num_heads=2, num_kv_heads=1, scalar=512.0, window=100), [10, 150], 90),
]


@pytest.mark.parametrize("name,over,prefixes,C", CASES, ids=[c[0] for c in CASES])
def test_chunk_matches_oracle(name, over, prefixes, C):
    layer = W.Layer(**{**BASE, **over})
    d, c = chunk_case(layer, prefixes, C, pad=37, seed=400 + len(name))
    out, st, dev = run_chunk(layer, d, c, prefixes)
    assert st == 0
    # the append wrote the chunk's rows, and nothing else
    kc_ref = c["k_cache"].clone()
    for b, p in enumerate(prefixes):
        kc_ref[b, p:p + C] = c["k_new"][b]
    assert torch.equal(dev["k_cache"].cpu(), kc_ref)
    kc = dev["k_cache"].cpu()
    vc = None if layer.k_eq_v else dev["v_cache"].cpu()
    ref = O.attention_prefill_chunk(c["q"], kc, vc, prefixes, layer, w_q=d["w_q"], w_k=d["w_k"])
    assert_close(out, ref, name)


def test_chunk_without_append_equals_with_append():
    layer = W.Layer(**{**BASE, "window": 50})
    prefixes, C = [9, 140], 70
    d, c = chunk_case(layer, prefixes, C, pad=5, seed=7)
    a, st_a, _ = run_chunk(layer, d, c, prefixes, append=True)
    b, st_b, _ = run_chunk(layer, d, c, prefixes, append=False)
    assert st_a == 0 and st_b == 0
    assert torch.equal(a, b)


@pytest.mark.parametrize("over", [dict(), dict(window=128, qk_norm=W.NORM_W)])
def test_whole_prompt_chunk_is_bit_identical_to_prefill(over):
    layer = W.Layer(**{**BASE, **over})
    S = 300
    gm = 1.0 if layer.qk_norm == W.NORM_W else 0.0
    d = small_prefill_inputs(layer, 2, S, seed=8, gain_mean=gm)
    L = make_layer(layer, S, d["w_q"], d["w_k"])
    dv = to_dev(d)
    ref = L.prefill(dv["q"], dv["k"], dv["v"], dv["positions"])
    pre = torch.zeros(2, dtype=torch.int32, device="cuda")
    got = L.prefill_chunk(dv["q"], dv["k"], dv["v"], pre)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)


def test_prompt_in_chunks_equals_whole_prompt():
    # a prompt fed as chunks of 128, 1, 200 and 71 tokens through the append gives the
    # whole-prompt prefill's rows and fills the cache with the prompt's rows
    layer = W.Layer(**{**BASE, "window": 150, "softcap": 30.0})
    sizes = [128, 1, 200, 71]
    S = sum(sizes)
    d = small_prefill_inputs(layer, 2, S, seed=9)
    L = make_layer(layer, S, d["w_q"], d["w_k"])
    dv = to_dev(d)
    whole = L.prefill(dv["q"], dv["k"], dv["v"], dv["positions"])
    kc = torch.zeros_like(dv["k"])
    vc = torch.zeros_like(dv["v"])
    outs, p = [], 0
    for n in sizes:
        pre = torch.full((2,), p, dtype=torch.int32, device="cuda")
        sl = slice(p, p + n)
        outs.append(L.prefill_chunk(dv["q"][:, sl].contiguous(), kc, vc, pre, k_new=dv["k"][:, sl].contiguous(),
                                    v_new=dv["v"][:, sl].contiguous()))
        p += n
    torch.cuda.synchronize()
    assert torch.equal(kc, dv["k"]) and torch.equal(vc, dv["v"])
    got = torch.cat(outs, dim=1)
    assert_close(got, whole.double().cpu().numpy(), "chunks vs whole")


def test_one_token_chunk_close_to_decode():
    layer = W.GEMMA4_DECODE_LOCAL.layer
    prefixes = [500, 1100]
    d, c = chunk_case(layer, prefixes, 1, pad=3, seed=10)
    out, st, dev = run_chunk(layer, d, c, prefixes)
    assert st == 0
    L = make_layer(layer, c["Lmax"], None, None)
    lens = torch.tensor([p + 1 for p in prefixes], dtype=torch.int32, device="cuda")
    dec = L.decode(dev["q"][:, 0].contiguous(), dev["k_cache"], dev["v_cache"], lens)
    torch.cuda.synchronize()
    assert_close(out[:, 0], dec.double().cpu().numpy(), "chunk of one vs decode")


def test_out_of_range_prefix_is_flagged_and_clamped():
    layer = W.Layer(**BASE)
    prefixes, C = [0, 60], 40
    d, c = chunk_case(layer, prefixes, C, pad=0, seed=11)   # Lmax = 100: 60 is the last legal prefix
    L = make_layer(layer, c["Lmax"], None, None)
    dev = {k: c[k].cuda().contiguous() for k in ("q", "k_new", "v_new", "k_cache", "v_cache")}
    ws = L.prefill_chunk_workspace(2, C, c["Lmax"])
    bad = torch.tensor([0, 75], dtype=torch.int32, device="cuda")
    L.prefill_chunk(dev["q"], dev["k_cache"], dev["v_cache"], bad, k_new=dev["k_new"], v_new=dev["v_new"],
                    workspace=ws)
    from gemma_family_decoder_b200 import check
    assert check(ws) == 6                                   # GATTN_ERR_DEVICE_BOUNDS


def test_chunk_workload_sampled_rows():
    # the benchmarked chunk (eight prompts' last 1024 tokens after 7168 cached) in the bench's
    # launch configuration: append + prologue + chunk kernel, sampled rows against the oracle
    wl = W.GEMMA3_GLOBAL_CHUNK
    d = W.chunk_inputs(wl)
    L = make_layer(wl.layer, d["max_len"], d["w_q"], d["w_k"])
    dev = {k: d[k].cuda().contiguous() for k in ("q", "k_new", "v_new", "k_cache", "v_cache", "prefix_lens")
           if d[k] is not None}
    ws = L.prefill_chunk_workspace(wl.batch, wl.chunk, d["max_len"])
    out = L.prefill_chunk(dev["q"], dev["k_cache"], dev.get("v_cache"), dev["prefix_lens"], k_new=dev["k_new"],
                          v_new=dev.get("v_new"), workspace=ws)
    from gemma_family_decoder_b200 import check
    assert check(ws) == 0
    rng = np.random.default_rng(wl.seed)
    rows = np.array(sorted({0, 1, 127, 128, 511, wl.chunk - 1} | set(int(r) for r in rng.integers(0, wl.chunk, 6))))
    kc = dev["k_cache"].cpu()
    vc = None if wl.layer.k_eq_v else dev["v_cache"].cpu()
    ref = O.attention_prefill_chunk(d["q"], kc, vc, d["prefix_lens"], wl.layer, w_q=d["w_q"], w_k=d["w_k"], rows=rows)
    assert_close(out[:, torch.as_tensor(rows, device=out.device)], ref, wl.name)
