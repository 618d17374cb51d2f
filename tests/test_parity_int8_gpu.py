"""GPU parity of the int8 KV cache: gattn_kv_quantize and gattn_decode_int8 (the persistent
CUDA-core kernel for 1, 2 or 4 query heads per kv head, the tensor-core kernel for K=V
layers with 8 or 16, the split kernel for the rest).

The quantiser is integer work decided by float32 division on both sides, so
its codes and scales must equal the oracle's bit for bit.  The int8 decode is
compared with the oracle's decode over the dequantised rows (max-abs 2e-2,
mean-abs 2e-3).  The caches are quantised by the library from bf16 rows; the
scales of rows a query never sees are then set to NaN, so a kernel that reads
one fails parity.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from helpers import assert_close, decode_full_cache, make_layer

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def quantize_dev(x):
    from gemma_family_decoder_b200 import kv_quantize
    codes, scales = kv_quantize(x.contiguous())
    torch.cuda.synchronize()
    return codes, scales


@pytest.mark.parametrize("D", [256, 512])
def test_kv_quantize_bit_exact(D):
    g = torch.Generator().manual_seed(D)
    x = (torch.randn(3, 37, 2, D, generator=g) * torch.rand(3, 37, 2, 1, generator=g) * 40).to(torch.bfloat16)
    x[0, 0, 0] = 0.0                                     # zero row: s = 0, codes 0
    x[0, 1, 1] = 0.0
    x[0, 1, 1, 7] = -3e-38                               # tiny row
    x[1, 2, 0, :8] = torch.tensor([0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 126.5, 127.0])  # exact halves
    x[1, 2, 0, 8:] = 0.0
    x[2, 3, 1] *= 1e30                                   # huge row
    codes, scales = quantize_dev(x.cuda())
    ref_c, ref_s = O.kv_quantize(x.float().numpy())
    assert np.array_equal(codes.cpu().numpy(), ref_c)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), ref_s.view(np.uint32))
    assert codes[1, 2, 0, :8].tolist() == [0, 2, 2, 0, -2, -2, 126, 127]


def test_kv_quantize_empty_and_ragged_row_count():
    from gemma_family_decoder_b200 import kv_quantize
    x = torch.randn(13, 256, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16).cuda()
    c, s = kv_quantize(x)                                # 13 rows: a partial block of 8
    rc, rs = O.kv_quantize(x.float().cpu().numpy())
    assert np.array_equal(c.cpu().numpy(), rc) and np.array_equal(s.cpu().numpy(), rs)
    e = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    c0, s0 = kv_quantize(e)
    assert c0.numel() == 0 and s0.numel() == 0


def int8_caches(wl, seq_lens, max_len=None, layer=None):
    """Device codes/scales (NaN scales outside the visible rows) and the oracle's own
    codes/scales of the visible rows, checked equal."""
    layer = layer or wl.layer
    k, v, oa = decode_full_cache(wl, seq_lens, max_len=max_len, layer=layer)
    kq, ks = quantize_dev(torch.nan_to_num(k))
    vq, vs = (None, None) if v is None else quantize_dev(torch.nan_to_num(v))
    B = len(seq_lens)
    host = dict(kc=[], ks=[], vc=[], vs=[], first_rows=oa["first_rows"])
    for b in range(B):
        lo, L = oa["first_rows"][b], int(seq_lens[b])
        ks[b, :lo] = float("nan")
        ks[b, L:] = float("nan")
        c, s = O.kv_quantize(oa["k_cache"][b].float().numpy())
        assert np.array_equal(kq[b, lo:L].cpu().numpy(), c)
        host["kc"].append(c)
        host["ks"].append(s)
        if v is not None:
            vs[b, :lo] = float("nan")
            vs[b, L:] = float("nan")
            c, s = O.kv_quantize(oa["v_cache"][b].float().numpy())
            assert np.array_equal(vq[b, lo:L].cpu().numpy(), c)
            host["vc"].append(c)
            host["vs"].append(s)
    return (kq, ks, vq, vs), host


def run_decode_int8(layer, q, dev, seq_lens, w_q, w_k):
    kq, ks, vq, vs = dev
    L = make_layer(layer, kq.shape[1], w_q, w_k)
    ws = L.decode_workspace(kq.shape[0], kq.shape[1])
    out = L.decode_int8(q.cuda(), kq, ks, vq, vs, seq_lens.cuda(), workspace=ws)
    from gemma_family_decoder_b200 import check
    return out, check(ws)


def oracle_int8(dq, host, seq_lens, layer, batches=None):
    return O.attention_decode_int8(dq["q"], host["kc"], host["ks"], host["vc"] or None, host["vs"] or None,
                                   seq_lens, layer, w_q=dq["w_q"], w_k=dq["w_k"], batches=batches,
                                   first_rows=host["first_rows"])


INT8_CASES = [
    ("local_gqa2_w1024", W.GEMMA4_DECODE_LOCAL.layer, [1, 2, 255, 256, 257, 1023, 1024, 1025, 3000]),
    ("g1_d512_keqv_r128_norm", W.Layer(num_heads=2, num_kv_heads=2, head_dim=512, rotary_fraction=0.25,
                                       scalar=512.0, k_eq_v=True, qk_norm=W.NORM_W), [1, 33, 700]),
    ("g2_d512_cap_w300_r256", W.Layer(num_heads=4, num_kv_heads=2, head_dim=512, softcap=50.0, window=300,
                                      rotary_fraction=0.5, scalar=512.0), [5, 299, 300, 301, 1000]),
    ("g2_d512_full_rope", W.Layer(num_heads=2, num_kv_heads=1, head_dim=512, rope_theta=1e6, scalar=512.0),
     [3, 77, 1030]),
    ("g4_d256_r64_norm1", W.Layer(num_heads=4, num_kv_heads=1, head_dim=256, rotary_fraction=0.25,
                                  qk_norm=W.NORM_ONE_PLUS_W), [2, 100, 513]),
    ("g4_d256_keqv_hkv4", W.Layer(num_heads=16, num_kv_heads=4, head_dim=256, rope_theta=1e6, k_eq_v=True),
     [7, 600]),
    ("g1_d256_norope_keqv_hkv8", W.Layer(num_heads=8, num_kv_heads=8, head_dim=256, rotary_fraction=0.0,
                                         k_eq_v=True), [1, 9, 64, 65]),
    ("g2_d256_r16_cap_w5", W.Layer(num_heads=8, num_kv_heads=4, head_dim=256, rotary_fraction=0.0625,
                                   softcap=30.0, window=5), [1, 4, 5, 6, 40]),
    # K=V with 8 or 16 query heads per kv head: the tensor-core kernel on the codes
    ("global_keqv_g16_d512", W.GEMMA4_DECODE_GLOBAL.layer, [1, 700, 2049, 2500]),
    ("keqv_g8_d512_norm", W.Layer(num_heads=8, num_kv_heads=1, head_dim=512, rope_theta=1e6, rotary_fraction=0.25,
                                  scalar=512.0, k_eq_v=True, qk_norm=W.NORM_W), [3, 65, 700]),
    ("keqv_g16_d512_norope", W.Layer(num_heads=16, num_kv_heads=1, head_dim=512, rotary_fraction=0.0,
                                     scalar=512.0, k_eq_v=True), [1, 128, 129, 2048, 4100]),
    ("keqv_g16_d256_cap_r16_norm1", W.Layer(num_heads=32, num_kv_heads=2, head_dim=256, rotary_fraction=0.0625,
                                            softcap=30.0, k_eq_v=True, qk_norm=W.NORM_ONE_PLUS_W, window=200),
     [1, 150, 199, 200, 201, 1300]),
    ("keqv_g8_d256_r64_w1000_norm", W.Layer(num_heads=8, num_kv_heads=1, head_dim=256, rotary_fraction=0.25,
                                            k_eq_v=True, qk_norm=W.NORM_W, window=1000), [999, 1000, 1001, 3333]),
    # 8 or 16 query heads per kv head without K=V: the CUDA-core split kernel
    ("g8_d256_window_cap", W.Layer(num_heads=16, num_kv_heads=2, head_dim=256, window=200, softcap=30.0),
     [1, 199, 200, 201, 900]),
]


@pytest.mark.parametrize("name,layer,lens", INT8_CASES, ids=[c[0] for c in INT8_CASES])
def test_decode_int8_small_matches_oracle(name, layer, lens):
    gm = 1.0 if layer.qk_norm == W.NORM_W else 0.0
    wl = W.DecodeWorkload(name, layer, len(lens), 1, max(lens), seed=21, gain_mean=gm)
    dq = W.decode_inputs(wl, layer=layer)
    seq_lens = torch.tensor(lens, dtype=torch.int32)
    dev, host = int8_caches(wl, seq_lens, max_len=max(lens) + 5, layer=layer)
    out, st = run_decode_int8(layer, dq["q"], dev, seq_lens, dq["w_q"], dq["w_k"])
    assert st == 0
    assert_close(out, oracle_int8(dq, host, seq_lens, layer), name)


def test_decode_int8_workload_matches_oracle():
    wl = W.GEMMA4_DECODE_LOCAL
    dq = W.decode_inputs(wl)
    seq_lens = dq["seq_lens"]
    dev, host = int8_caches(wl, seq_lens)
    out, st = run_decode_int8(wl.layer, dq["q"], dev, seq_lens, dq["w_q"], dq["w_k"])
    assert st == 0
    assert_close(out, oracle_int8(dq, host, seq_lens, wl.layer), wl.name + " int8")


@pytest.mark.parametrize("wl", [W.GEMMA4_DECODE_GLOBAL, W.GEMMA4_DECODE_GLOBAL_NORM], ids=lambda w: w.name)
def test_decode_int8_global_workload_matches_oracle(wl):
    # the Gemma 4 global K=V layer over a full-size int8 cache (the tensor-core kernel), every
    # fourth batch row against the oracle
    dq = W.decode_inputs(wl)
    seq_lens = dq["seq_lens"]
    k, v, oa = decode_full_cache(wl, seq_lens)
    kq, ks = quantize_dev(torch.nan_to_num(k))
    del k, v
    batches = list(range(0, wl.batch, 4))
    kc = [None] * wl.batch
    ksc = [None] * wl.batch
    for b in batches:
        L = int(seq_lens[b])
        kc[b], ksc[b] = O.kv_quantize(oa["k_cache"][b].float().numpy())
        assert np.array_equal(kq[b, :L].cpu().numpy(), kc[b])
        ks[b, L:] = float("nan")
    out, st = run_decode_int8(wl.layer, dq["q"], (kq, ks, None, None), seq_lens, dq["w_q"], dq["w_k"])
    assert st == 0
    ref = O.attention_decode_int8(dq["q"], kc, ksc, None, None, seq_lens, wl.layer, w_q=dq["w_q"], w_k=dq["w_k"],
                                  batches=batches)
    assert_close(out[batches], ref, wl.name + " int8")


def test_decode_int8_tensor_core_zero_rows():
    # zero rows (scale 0, codes 0) in a K=V layer on the tensor-core kernel: ordinary keys
    # with logit 0 and value 0, under QK-norm (their norm is sqrt(eps))
    layer = W.GEMMA4_DECODE_GLOBAL_NORM.layer
    wl = W.DecodeWorkload("z16", layer, 2, 1, 700, seed=29, gain_mean=1.0, gain_std=0.1)
    dq = W.decode_inputs(wl)
    seq_lens = torch.tensor([700, 333], dtype=torch.int32)
    k, v, oa = decode_full_cache(wl, seq_lens, max_len=700)
    k = torch.nan_to_num(k)
    k[0, 10:20] = 0.0
    k[1, 128:300] = 0.0
    kq, ks = quantize_dev(k)
    out, st = run_decode_int8(layer, dq["q"], (kq, ks, None, None), seq_lens, dq["w_q"], dq["w_k"])
    assert st == 0
    kd = [O.kv_dequantize(*O.kv_quantize(k[b, :int(seq_lens[b])].float().cpu().numpy())) for b in range(2)]
    ref = O.attention_decode(dq["q"], kd, None, seq_lens, layer, w_q=dq["w_q"], w_k=dq["w_k"])
    assert_close(out, ref, "zero rows, tensor core")


def test_decode_int8_zero_rows_and_bad_length():
    # zero cache rows (scale 0) are ordinary keys with logit 0; a bad length is flagged and zeroed
    layer = W.GEMMA4_DECODE_LOCAL.layer
    wl = W.DecodeWorkload("z", layer, 2, 1, 300, seed=23)
    dq = W.decode_inputs(wl)
    seq_lens = torch.tensor([300, 200], dtype=torch.int32)
    k, v, oa = decode_full_cache(wl, seq_lens, max_len=300)
    k = torch.nan_to_num(k)
    v = torch.nan_to_num(v)
    k[0, 10:20] = 0.0
    v[0, 15:40] = 0.0
    kq, ks = quantize_dev(k)
    vq, vs = quantize_dev(v)
    out, st = run_decode_int8(layer, dq["q"], (kq, ks, vq, vs), seq_lens, None, None)
    assert st == 0
    kd = [O.kv_dequantize(*O.kv_quantize(k[b, :int(seq_lens[b])].float().cpu().numpy())) for b in range(2)]
    vd = [O.kv_dequantize(*O.kv_quantize(v[b, :int(seq_lens[b])].float().cpu().numpy())) for b in range(2)]
    ref = O.attention_decode(dq["q"], kd, vd, seq_lens, layer)
    assert_close(out, ref, "zero rows")
    bad = torch.tensor([0, 200], dtype=torch.int32)
    out2, st2 = run_decode_int8(layer, dq["q"], (kq, ks, vq, vs), bad, None, None)
    assert st2 == 6
    assert torch.count_nonzero(out2[0]) == 0
    assert_close(out2[1:], ref[1:], "bad length, other row")
