"""GPU parity of the padded-batch prefill (gattn_prefill_padded) against the oracle.

A padded batch gives each sequence's valid tokens [lo, hi) (the batched-prompt
attention_mask of KerasFormers "Gemma 4", Gemma4Generate.generate).  Valid tokens
take positions 0, 1, ... from lo, as a left-padded prompt numbers them; padding
tokens take position 0 (they are rotated, then ignored).  Padding rows must come
out exactly zero, even in an output buffer that held NaN.
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


def padded_positions(S, ranges):
    pos = torch.zeros(len(ranges), S, dtype=torch.int32)
    for b, (lo, hi) in enumerate(ranges):
        if hi > lo:
            pos[b, lo:hi] = torch.arange(hi - lo, dtype=torch.int32)
    return pos


def run_padded(d, ranges, max_pos=None):
    layer = d["layer"]
    B, S = d["q"].shape[:2]
    L = make_layer(layer, max_pos or max(S, 1), d["w_q"], d["w_k"])
    dv = to_dev(d)
    sr = torch.tensor(ranges, dtype=torch.int32, device="cuda").reshape(B, 2)
    out = torch.full_like(dv["q"], float("nan"))
    ws = L.prefill_workspace(B, S)
    L.prefill(dv["q"], dv["k"], dv["v"], dv["positions"], out=out, workspace=ws, seq_range=sr)
    from gemma_family_decoder_b200 import check
    st = check(ws)
    torch.cuda.synchronize()
    return out, st


def padded_inputs(layer, ranges, S, seed):
    gm = 1.0 if layer.qk_norm == W.NORM_W else 0.0
    d = small_prefill_inputs(layer, len(ranges), S, seed=seed, gain_mean=gm)
    d["positions"] = padded_positions(S, ranges)
    return d


def check_padding_rows_zero(out, ranges):
    S = out.shape[1]
    for b, (lo, hi) in enumerate(ranges):
        pad = torch.ones(S, dtype=torch.bool)
        if hi > lo:
            pad[lo:hi] = False
        rows = out[b, pad.cuda()]
        assert torch.isfinite(rows.float()).all(), f"batch {b}: padding rows not written"
        assert torch.count_nonzero(rows) == 0, f"batch {b}: padding rows not zero"


BASE = dict(num_heads=4, num_kv_heads=2, head_dim=256, scalar=256.0)
S0 = 300
# (name, layer overrides, S, per-sequence [lo, hi))
CASES = [
    ("left", dict(), S0, [(37, S0), (0, S0)]),
    ("right", dict(), S0, [(0, S0 - 70), (0, 5)]),
    # lo >= 128: the first query tile is all padding; lo = hi and [0, 0): no valid token
    ("mixed", dict(), S0, [(130, S0), (5, 150), (S0, S0), (0, 0)]),
    ("one_token", dict(num_kv_heads=1), 200, [(199, 200), (0, 1), (64, 65)]),
    ("window7_left", dict(window=7), S0, [(100, S0), (3, 260)]),
    ("window128_softcap", dict(window=128, softcap=50.0), 400, [(129, 400), (0, 257)]),
    ("window_gt_S", dict(window=500), S0, [(11, 290)]),
    ("gqa8_qknorm", dict(num_heads=8, num_kv_heads=1, qk_norm=W.NORM_ONE_PLUS_W), 260, [(60, 260), (0, 200)]),
    ("keqv_partial", dict(k_eq_v=True, rotary_fraction=0.5), 190, [(17, 190), (0, 100)]),
    ("d512_keqv", dict(head_dim=512, num_heads=4, num_kv_heads=1, k_eq_v=True, rotary_fraction=0.25,
                       rope_theta=1e6, qk_norm=W.NORM_W, scalar=512.0), 200, [(70, 200), (0, 131)]),
    ("d512_window", dict(head_dim=512, num_heads=2, num_kv_heads=1, scalar=512.0, window=100), 150,
     [(65, 150), (0, 64)]),
]


@pytest.mark.parametrize("name,over,S,ranges", CASES, ids=[c[0] for c in CASES])
def test_padded_prefill_matches_oracle(name, over, S, ranges):
    layer = W.Layer(**{**BASE, **over})
    d = padded_inputs(layer, ranges, S, seed=300 + len(name))
    out, st = run_padded(d, ranges)
    assert st == 0
    ref = O.attention_prefill(d["q"], d["k"], d["v"], d["positions"], layer, w_q=d["w_q"], w_k=d["w_k"],
                              seq_range=ranges)
    assert_close(out, ref, name)
    check_padding_rows_zero(out, ranges)


# head_dim 512 with an odd number of query heads per kv head: whole prompts and
# padded batches run the same single-SM kernel (even groups take the SM-pair
# kernel for whole prompts, equal to the padded path within rounding:
# test_parity_pair_gpu.py)
@pytest.mark.parametrize("over,S", [(dict(), 300), (dict(window=128), 257),
                                    (dict(head_dim=512, num_heads=3, num_kv_heads=1, scalar=512.0), 130)])
def test_full_ranges_bit_identical_to_unpadded(over, S):
    layer = W.Layer(**{**BASE, **over})
    d = small_prefill_inputs(layer, 2, S, seed=41)
    L = make_layer(layer, S, d["w_q"], d["w_k"])
    dv = to_dev(d)
    ref = L.prefill(dv["q"], dv["k"], dv["v"], dv["positions"])
    sr = torch.tensor([[0, S], [0, S]], dtype=torch.int32, device="cuda")
    got = L.prefill(dv["q"], dv["k"], dv["v"], dv["positions"], seq_range=sr)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)


@pytest.mark.parametrize("Wn", [0, 50])
def test_left_padded_equals_sequence_alone(Wn):
    # the valid rows of a left-padded sequence are the prefill of that sequence alone
    layer = W.Layer(**{**BASE, "window": Wn})
    n, p = 200, 90
    d = small_prefill_inputs(layer, 1, n, seed=43)
    L = make_layer(layer, n, d["w_q"], d["w_k"])
    dv = to_dev(d)
    alone = L.prefill(dv["q"], dv["k"], dv["v"], dv["positions"])
    S = n + p

    def pad(x):
        z = torch.randn((1, p) + tuple(x.shape[2:]), generator=torch.Generator().manual_seed(7))
        return torch.cat([z.to(x.dtype).cuda(), x], dim=1).contiguous()

    pos = torch.cat([torch.zeros(1, p, dtype=torch.int32).cuda(), dv["positions"]], dim=1).contiguous()
    sr = torch.tensor([[p, S]], dtype=torch.int32, device="cuda")
    got = L.prefill(pad(dv["q"]), pad(dv["k"]), pad(dv["v"]), pos, seq_range=sr)
    torch.cuda.synchronize()
    assert torch.count_nonzero(got[:, :p]) == 0
    assert_close(got[:, p:], alone.double().cpu().numpy(), "left padded vs alone")


@pytest.mark.parametrize("Wn,lo,hi", [(0, 40, 250), (0, 129, 256), (9, 3, 200), (128, 130, 256)])
def test_padded_mask_is_exact(Wn, lo, hi):
    # q = 0: uniform weights over the visible keys; one-hot values name them
    S, D = 256, 256
    layer = W.Layer(num_heads=2, num_kv_heads=1, head_dim=D, window=Wn, rotary_fraction=1.0)
    q = torch.zeros(1, S, 2, D, dtype=torch.bfloat16)
    k = torch.randn(1, S, 1, D, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    v = torch.zeros(1, S, 1, D, dtype=torch.bfloat16)
    v[0, torch.arange(S), 0, torch.arange(S)] = 1.0
    d = dict(q=q, k=k, v=v, positions=padded_positions(S, [(lo, hi)]), w_q=None, w_k=None, layer=layer)
    out, st = run_padded(d, [(lo, hi)])
    assert st == 0
    got = out[0].float().cpu().numpy()
    for i in range(S):
        vis = np.zeros(D, dtype=bool)
        if lo <= i < hi:
            first = lo if Wn == 0 else max(lo, i - Wn + 1)
            vis[first:i + 1] = True
        for hh in range(2):
            nz = got[i, hh] != 0
            assert np.array_equal(nz, vis), (i, hh)
            if vis.any():
                np.testing.assert_allclose(got[i, hh, vis], 1.0 / vis.sum(), rtol=1e-2)


def test_out_of_range_seq_range_is_flagged_and_clamped():
    layer = W.Layer(num_heads=2, num_kv_heads=1, head_dim=256)
    S = 140
    ranges = [(-5, 60), (20, S + 9)]
    d = padded_inputs(layer, [(0, 60), (20, S)], S, seed=17)
    out, st = run_padded(d, ranges)
    assert st == 6                   # GATTN_ERR_DEVICE_BOUNDS
    clamped = [(0, 60), (20, S)]
    ref = O.attention_prefill(d["q"], d["k"], d["v"], d["positions"], layer, seq_range=clamped)
    assert_close(out, ref, "clamped")
    check_padding_rows_zero(out, clamped)


def test_leftpad_workload_sampled_rows():
    # the benchmarked left-padded batch at full size: rows on both sides of every
    # sequence's first kept token, the first and last tiles, and random rows
    wl = W.GEMMA3_GLOBAL_LEFTPAD
    d = W.prefill_inputs(wl)
    ranges = d["seq_range"].tolist()
    S = wl.seq
    L = make_layer(wl.layer, S, d["w_q"], d["w_k"])
    dv = to_dev(d, keys=("q", "k", "v", "positions", "seq_range"))
    ws = L.prefill_workspace(wl.batch, S)
    out = L.prefill(dv["q"], dv["k"], dv["v"], dv["positions"], workspace=ws, seq_range=dv["seq_range"])
    from gemma_family_decoder_b200 import check
    assert check(ws) == 0
    torch.cuda.synchronize()
    rng = np.random.default_rng(wl.seed)
    rows = {0, 127, 128, S - 129, S - 1} | set(int(r) for r in rng.integers(0, S, 6))
    for lo, _ in ranges:
        rows |= {max(0, lo - 1), lo, min(S - 1, lo + 1), min(S - 1, lo + 200)}
    rows = np.array(sorted(rows))
    ref = O.attention_prefill(d["q"], d["k"], d["v"], d["positions"], wl.layer, w_q=d["w_q"], w_k=d["w_k"],
                              rows=rows, seq_range=ranges)
    got = out[:, torch.as_tensor(rows, device=out.device)]
    assert_close(got, ref, wl.name)
    check_padding_rows_zero(out, ranges)
