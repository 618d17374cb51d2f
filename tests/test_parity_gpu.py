"""GPU parity: libgattn (through its C ABI) against the float64 oracle.

Small cases compare every output element; the full-size workloads compare the
rows (prefill) or batch rows (decode) the oracle can afford.  Tolerance for
bf16 inputs with fp32 accumulation: max-abs 2e-2 and mean-abs 2e-3.  The
integer mask is checked exactly with the one-hot probe.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from helpers import (assert_close, decode_full_cache, err_stats, make_layer,
                     small_prefill_inputs, to_dev)

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def run_prefill(d, max_pos=None):
    layer = d["layer"]
    S = d["q"].shape[1]
    L = make_layer(layer, max_pos or max(S, 1), d["w_q"], d["w_k"])
    dv = to_dev(d)
    out = L.prefill(dv["q"], dv["k"], dv["v"], dv["positions"])
    ws = L.prefill_workspace(d["q"].shape[0], S)
    out2 = L.prefill(dv["q"], dv["k"], dv["v"], dv["positions"], workspace=ws)
    from gemma_family_decoder_b200 import check
    assert check(ws) == 0
    torch.cuda.synchronize()
    return out, out2


def oracle_prefill(d, rows=None):
    return O.attention_prefill(d["q"], d["k"], d["v"], d["positions"], d["layer"],
                               w_q=d["w_q"], w_k=d["w_k"], rows=rows)


BASE = dict(num_heads=4, num_kv_heads=2, head_dim=256, scalar=256.0)
SMALL_CASES = [
    # (name, layer overrides, B, S)
    ("causal_s1", dict(), 1, 1),
    ("causal_s3", dict(), 2, 3),
    ("causal_s17", dict(), 1, 17),
    ("causal_s129_ragged", dict(), 2, 129),
    ("causal_s300", dict(num_kv_heads=1), 1, 300),
    ("window1", dict(window=1), 1, 130),
    ("window5", dict(window=5), 1, 200),
    ("window128_softcap", dict(window=128, softcap=50.0), 1, 384),
    ("window_S_plus_3", dict(window=300), 1, 297),
    ("gqa8_theta1e6", dict(num_heads=8, num_kv_heads=1, rope_theta=1e6), 1, 260),
    ("qknorm_one_plus_w", dict(qk_norm=W.NORM_ONE_PLUS_W, window=64), 2, 200),
    ("qknorm_w_partial", dict(qk_norm=W.NORM_W, rotary_fraction=0.25), 1, 150),
    ("no_rope", dict(rotary_fraction=0.0), 1, 140),
    ("keqv_d256", dict(k_eq_v=True, rotary_fraction=0.5), 1, 190),
    ("mha_hkv_eq_h", dict(num_heads=2, num_kv_heads=2, softcap=10.0), 1, 257),
    ("d512_keqv_partial_norm", dict(head_dim=512, num_heads=4, num_kv_heads=1, k_eq_v=True,
                                    rotary_fraction=0.25, rope_theta=1e6, qk_norm=W.NORM_W,
                                    scalar=512.0), 1, 200),
    ("d512_separate_v", dict(head_dim=512, num_heads=2, num_kv_heads=1, scalar=512.0,
                             window=100), 1, 150),
]


@pytest.mark.parametrize("name,over,B,S", SMALL_CASES, ids=[c[0] for c in SMALL_CASES])
def test_prefill_small_matches_oracle(name, over, B, S):
    layer = W.Layer(**{**BASE, **over})
    gm = 1.0 if layer.qk_norm == W.NORM_W else 0.0
    d = small_prefill_inputs(layer, B, S, seed=100 + len(name), gain_mean=gm)
    out, out2 = run_prefill(d)
    assert_close(out, oracle_prefill(d), name)
    # deterministic: the same call twice is bit-identical
    assert torch.equal(out, out2)


@pytest.mark.parametrize("S,Wn", [(64, 0), (200, 0), (200, 1), (200, 7), (256, 128), (256, 255), (129, 300)])
def test_prefill_mask_is_exact(S, Wn):
    # q = 0 -> uniform weights over the visible keys; one-hot values read them out
    D = 256
    layer = W.Layer(num_heads=2, num_kv_heads=1, head_dim=D, window=Wn, rotary_fraction=1.0)
    q = torch.zeros(1, S, 2, D, dtype=torch.bfloat16)
    k = torch.randn(1, S, 1, D, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    v = torch.zeros(1, S, 1, D, dtype=torch.bfloat16)
    n = min(S, D)
    v[0, torch.arange(n), 0, torch.arange(n)] = 1.0
    d = dict(q=q, k=k, v=v, positions=torch.arange(S, dtype=torch.int32)[None], w_q=None, w_k=None,
             layer=layer)
    out, _ = run_prefill(d)
    got = out[0, :, :, :n].float().cpu().numpy()
    for i in range(S):
        lo = 0 if Wn == 0 else max(0, i - Wn + 1)
        vis = np.zeros(n, dtype=bool)
        vis[lo:min(i + 1, n)] = True
        for hh in range(2):
            nz = got[i, hh] != 0
            assert np.array_equal(nz, vis), (i, hh)
    # and the weights are 1/|V_i| to bf16 rounding
    ref = oracle_prefill(d)[0, :, :, :n]
    assert np.max(np.abs(got - ref)) < 4e-3


def test_keqv_null_v_equals_passing_k():
    layer = W.Layer(num_heads=4, num_kv_heads=1, head_dim=512, k_eq_v=True, rotary_fraction=0.25,
                    rope_theta=1e6, qk_norm=W.NORM_W, scalar=512.0)
    d = small_prefill_inputs(layer, 1, 140, seed=7, gain_mean=1.0)
    out_null, _ = run_prefill(d)
    L = make_layer(layer, 140, d["w_q"], d["w_k"])
    dv = to_dev(d)
    out_k = L.prefill(dv["q"], dv["k"], dv["k"], dv["positions"])
    torch.cuda.synchronize()
    assert torch.equal(out_null, out_k)


def test_mqa_equals_replicated_gqa_on_gpu():
    base = W.Layer(num_heads=8, num_kv_heads=1, head_dim=256, window=50)
    d = small_prefill_inputs(base, 1, 160, seed=8)
    out_mqa, _ = run_prefill(d)
    for hkv in (2, 4, 8):
        rep = dict(d, k=d["k"].repeat(1, 1, hkv, 1), v=d["v"].repeat(1, 1, hkv, 1),
                   layer=dataclasses.replace(base, num_kv_heads=hkv))
        out_rep, _ = run_prefill(rep)
        # each (head, query tile) sees the same keys and values: bit-identical
        assert torch.equal(out_mqa, out_rep), hkv


# --- the workloads at full size ---------------------------------------------------

def sample_rows(S, n_rand=24, seed=0):
    rng = np.random.default_rng(seed)
    rows = set(range(0, min(S, 130))) | set(range(max(0, S - 130), S))
    rows |= set(int(r) for r in rng.integers(0, S, n_rand))
    return np.array(sorted(rows))


@pytest.mark.parametrize("wl", [W.GEMMA2_LOCAL, W.GEMMA1_MQA, W.GEMMA3_LOCAL, W.GEMMA3_GLOBAL],
                         ids=lambda w: w.name)
def test_prefill_workload_matches_oracle(wl):
    d = W.prefill_inputs(wl)
    out, _ = run_prefill(d)
    S = wl.seq
    rows = None if S <= 256 else sample_rows(S, seed=wl.seed)
    ref = oracle_prefill(d, rows=rows)
    got = out if rows is None else out[:, torch.as_tensor(rows, device=out.device)]
    assert_close(got, ref, wl.name)


def test_prefill_gemma4_global_sampled_rows():
    wl = W.GEMMA4_GLOBAL
    d = W.prefill_inputs(wl)
    out, _ = run_prefill(d)
    rng = np.random.default_rng(3)
    rows = np.array(sorted(set([0, 1, 127, 128, 4095, 16384, wl.seq - 129, wl.seq - 1]) |
                           set(int(r) for r in rng.integers(0, wl.seq, 8))))
    ref = oracle_prefill(d, rows=rows)
    got = out[:, torch.as_tensor(rows, device=out.device)]
    assert_close(got, ref, wl.name)


# --- decode ---------------------------------------------------------------------------

def run_decode(layer, wl, q, k, v, seq_lens, w_q, w_k):
    L = make_layer(layer, k.shape[1], w_q, w_k)
    ws = L.decode_workspace(k.shape[0], k.shape[1])
    out = L.decode(q.cuda(), k.cuda().contiguous(), None if v is None else v.cuda().contiguous(),
                   seq_lens.cuda(), workspace=ws)
    from gemma_family_decoder_b200 import check
    st = check(ws)
    return out, st


DEC_CASES = [
    ("local_gqa2_w1024", W.GEMMA4_DECODE_LOCAL.layer, [1, 2, 255, 256, 257, 1023, 1024, 1025, 3000]),
    ("global_keqv_d512", W.GEMMA4_DECODE_GLOBAL.layer, [1, 17, 1024, 1025, 2049, 3000]),
    ("global_keqv_qknorm", W.GEMMA4_DECODE_GLOBAL_NORM.layer, [5, 1500, 2048]),
    ("mqa_d256_softcap_norm1", W.Layer(num_heads=8, num_kv_heads=1, head_dim=256, softcap=50.0,
                                       qk_norm=W.NORM_ONE_PLUS_W, window=300), [1, 299, 300, 301, 900]),
    ("gqa4_d256", W.Layer(num_heads=16, num_kv_heads=4, head_dim=256, rope_theta=1e6), [7, 600]),
    # persistent CUDA-core split kernel (1, 2 or 4 query heads per kv head): every
    # RoPE branch (none, partner lane R/8 away, one or two same-lane groups),
    # both norm modes, softcap, window, K=V, head_dim 512, 1/2/4/8 kv heads
    ("simt_g1_d512_keqv_r128_norm", W.Layer(num_heads=2, num_kv_heads=2, head_dim=512,
                                            rotary_fraction=0.25, scalar=512.0, k_eq_v=True,
                                            qk_norm=W.NORM_W), [1, 33, 700]),
    ("simt_g2_d512_cap_w300_r256", W.Layer(num_heads=4, num_kv_heads=2, head_dim=512, softcap=50.0,
                                           window=300, rotary_fraction=0.5, scalar=512.0),
     [5, 299, 300, 301, 1000]),
    ("simt_g2_d512_full_rope", W.Layer(num_heads=2, num_kv_heads=1, head_dim=512, rope_theta=1e6,
                                       scalar=512.0), [3, 77, 1030]),
    ("simt_g4_d256_r64_norm1", W.Layer(num_heads=4, num_kv_heads=1, head_dim=256, rotary_fraction=0.25,
                                       qk_norm=W.NORM_ONE_PLUS_W), [2, 100, 513]),
    ("simt_g1_d256_norope_keqv", W.Layer(num_heads=8, num_kv_heads=8, head_dim=256,
                                         rotary_fraction=0.0, k_eq_v=True), [1, 9, 64, 65]),
    ("simt_g2_d256_r16_cap_w5", W.Layer(num_heads=8, num_kv_heads=4, head_dim=256, rotary_fraction=0.0625,
                                        softcap=30.0, window=5), [1, 4, 5, 6, 40]),
    # tensor-core split kernel (K=V, 8 or 16 query heads per kv head, <= 128 rotated dims)
    ("keqv_g8_d512_norm", W.Layer(num_heads=8, num_kv_heads=1, head_dim=512, rope_theta=1e6,
                                  rotary_fraction=0.25, scalar=512.0, k_eq_v=True,
                                  qk_norm=W.NORM_W), [3, 64, 65, 700]),
    ("keqv_g16_d256_cap_r16", W.Layer(num_heads=32, num_kv_heads=2, head_dim=256,
                                      rotary_fraction=0.0625, softcap=30.0, k_eq_v=True,
                                      qk_norm=W.NORM_ONE_PLUS_W, window=200),
     [1, 150, 199, 200, 201, 1300]),
    ("keqv_g16_d512_w512", W.Layer(num_heads=16, num_kv_heads=1, head_dim=512, window=512,
                                   rotary_fraction=0.25, scalar=512.0, k_eq_v=True),
     [100, 513, 2000]),
    # no rotation and no norm: the key warps touch only a chunk's ragged last
    # tile; several full chunks of 2048 keys stream through the ring
    ("keqv_g16_d512_norope", W.Layer(num_heads=16, num_kv_heads=1, head_dim=512, rotary_fraction=0.0,
                                     scalar=512.0, k_eq_v=True), [1, 128, 129, 2048, 4100]),
    ("keqv_g8_d256_r64_w1000", W.Layer(num_heads=8, num_kv_heads=1, head_dim=256, rotary_fraction=0.25,
                                       k_eq_v=True, qk_norm=W.NORM_W, window=1000), [999, 1000, 1001, 3333]),
    ("keqv_g16_d512_r32_norm1", W.Layer(num_heads=16, num_kv_heads=1, head_dim=512, rotary_fraction=0.0625,
                                        scalar=512.0, k_eq_v=True, qk_norm=W.NORM_ONE_PLUS_W), [257, 1999, 6000]),
]


@pytest.mark.parametrize("name,layer,lens", DEC_CASES, ids=[c[0] for c in DEC_CASES])
def test_decode_small_matches_oracle(name, layer, lens):
    gm = 1.0 if layer.qk_norm == W.NORM_W else 0.0
    wl = W.DecodeWorkload(name, layer, len(lens), 1, max(lens), seed=11, gain_mean=gm)
    dq = W.decode_inputs(wl, layer=layer)
    seq_lens = torch.tensor(lens, dtype=torch.int32)
    k, v, oa = decode_full_cache(wl, seq_lens, max_len=max(lens) + 5)
    out, st = run_decode(layer, wl, dq["q"], k, v, seq_lens, dq["w_q"], dq["w_k"])
    assert st == 0
    ref = O.attention_decode(dq["q"], oa["k_cache"], oa["v_cache"], seq_lens, layer,
                             w_q=dq["w_q"], w_k=dq["w_k"], first_rows=oa["first_rows"])
    assert_close(out, ref, name)


@pytest.mark.parametrize("wl", [W.GEMMA4_DECODE_LOCAL, W.GEMMA4_DECODE_GLOBAL, W.GEMMA4_DECODE_GLOBAL_NORM],
                         ids=lambda w: w.name)
def test_decode_workload_matches_oracle(wl):
    dq = W.decode_inputs(wl)
    seq_lens = dq["seq_lens"]
    k, v, oa = decode_full_cache(wl, seq_lens)
    out, st = run_decode(wl.layer, wl, dq["q"], k, v, seq_lens, dq["w_q"], dq["w_k"])
    assert st == 0
    batches = list(range(0, wl.batch, 4)) if wl.layer.window == 0 else list(range(wl.batch))
    ref = O.attention_decode(dq["q"], oa["k_cache"], oa["v_cache"], seq_lens, wl.layer,
                             w_q=dq["w_q"], w_k=dq["w_k"], batches=batches,
                             first_rows=oa["first_rows"])
    assert_close(out[torch.as_tensor(batches, device=out.device)], ref, wl.name)


def test_decode_equals_last_prefill_row_on_gpu():
    layer = W.Layer(num_heads=8, num_kv_heads=2, head_dim=256, window=100, qk_norm=W.NORM_W)
    d = small_prefill_inputs(layer, 2, 333, seed=12, gain_mean=1.0)
    pre, _ = run_prefill(d)
    q = d["q"][:, -1].contiguous()
    seq_lens = torch.full((2,), 333, dtype=torch.int32)
    dec, st = run_decode(layer, None, q, d["k"], d["v"], seq_lens, d["w_q"], d["w_k"])
    assert st == 0
    mx, mean = err_stats(dec, pre[:, -1].double().cpu().numpy())
    assert mx <= 2e-2 and mean <= 2e-3


# --- device-side checks and bounded waits -------------------------------------------

def test_bounded_wait_times_out_cleanly():
    from gemma_family_decoder_b200 import check, selftest_wait_timeout
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    selftest_wait_timeout(ws, 2000)
    assert check(ws) == 5           # GATTN_ERR_TIMEOUT
    assert check(ws) == 0           # cleared
    # the context is still usable
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0


def test_out_of_range_position_is_flagged():
    layer = W.Layer(num_heads=2, num_kv_heads=1, head_dim=256)
    d = small_prefill_inputs(layer, 1, 40, seed=13)
    L = make_layer(layer, 16)    # table shorter than the positions used
    dv = to_dev(d)
    ws = L.prefill_workspace(1, 40)
    L.prefill(dv["q"], dv["k"], dv["v"], dv["positions"], workspace=ws)
    from gemma_family_decoder_b200 import check
    assert check(ws) == 6           # GATTN_ERR_DEVICE_BOUNDS


def test_decode_bad_length_is_flagged_and_zeroed():
    layer = W.GEMMA4_DECODE_LOCAL.layer
    wl = W.DecodeWorkload("bad", layer, 2, 1, 64, seed=14)
    dq = W.decode_inputs(wl)
    seq_lens = torch.tensor([0, 64], dtype=torch.int32)
    k, v, _ = decode_full_cache(wl, torch.tensor([1, 64]), max_len=64)
    out, st = run_decode(layer, wl, dq["q"], torch.nan_to_num(k), torch.nan_to_num(v), seq_lens, None, None)
    assert st == 6
    assert torch.count_nonzero(out[0]) == 0
    assert torch.isfinite(out[1].float()).all()
