"""The work counts behind bench.py's numbers, against brute force on small shapes.

Every reported TFLOP/s and GB/s divides one of these counts by a time, so each is
checked here against an explicit enumeration: visible (query, key) pairs from the
mask itself, padded and chunked FLOPs from per-sequence masks, decode bytes from
the rows each query reads.
"""
import os
import sys

import numpy as np
import pytest
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
import workloads as W  # noqa: E402


def mask(S, window, lo=0, hi=None, q_off=0, n_keys=None):
    """Visible pairs by enumeration: query token q_off + i, key token j, within [lo, hi)."""
    hi = S if hi is None else hi
    n_keys = S if n_keys is None else n_keys
    i = q_off + np.arange(S)[:, None]
    j = np.arange(n_keys)[None, :]
    m = (j <= i) & (j >= lo) & (i >= lo) & (i < hi)
    if window > 0:
        m &= (i - j) < window
    return m


@pytest.mark.parametrize("S,Wn", [(1, 0), (7, 0), (300, 0), (300, 1), (300, 128), (300, 299), (300, 300), (300, 512)])
def test_visible_pairs_and_rows(S, Wn):
    m = mask(S, Wn)
    assert bench.visible_pairs(S, Wn) == int(m.sum())
    rows = np.arange(S)
    assert np.array_equal(bench.row_visible(rows, Wn), m.sum(axis=1))


def test_prefill_flops_whole_and_padded():
    L = W.Layer(num_heads=4, num_kv_heads=1, head_dim=256, window=50)
    wl = W.PrefillWorkload("t", L, 3, 200, 0)
    per_pair = 4.0 * 256 * 4
    assert bench.prefill_flops(wl) == per_pair * 3 * mask(200, 50).sum()
    sr = torch.tensor([[0, 200], [37, 200], [10, 120]], dtype=torch.int32)
    ref = sum(mask(200, 50, lo, hi).sum() for lo, hi in sr.tolist())
    assert bench.prefill_flops(wl, sr) == per_pair * ref
    # rows_flops: a row subset of a padded batch counts each sequence's kept rows only
    rows = np.array([0, 5, 36, 37, 119, 150, 199])
    d = dict(seq_range=sr)
    ref_rows = sum(mask(200, 50, lo, hi)[rows].sum() for lo, hi in sr.tolist())
    assert bench.rows_flops(wl, d, rows) == per_pair * ref_rows
    assert bench.rows_flops(wl, dict(seq_range=None), rows) == per_pair * 3 * mask(200, 50)[rows].sum()


@pytest.mark.parametrize("Wn", [0, 300])
def test_chunk_flops(Wn):
    L = W.Layer(num_heads=4, num_kv_heads=1, head_dim=256, window=Wn)
    wl = W.ChunkWorkload("c", L, 2, prefix=700, chunk=130, seed=0)
    m = mask(130, Wn, q_off=700, n_keys=830, hi=830)
    assert bench.chunk_flops(wl) == 4.0 * 256 * 4 * 2 * m.sum()
    rows = np.array([0, 64, 129])
    assert bench.chunk_flops(wl, rows) == 4.0 * 256 * 4 * 2 * m[rows].sum()


@pytest.mark.parametrize("int8", [False, True])
def test_decode_bytes(int8):
    L = W.Layer(num_heads=16, num_kv_heads=8, head_dim=256, window=1024)
    lens = np.array([1, 500, 1024, 1025, 30000])
    rows = sum(min(n, 1024) for n in lens)
    per_row = 8 * (256 + 4) if int8 else 8 * 256 * 2           # codes + one fp32 scale per kv head
    qo = len(lens) * 16 * 256 * 2 * 2
    assert bench.decode_bytes(L, lens, int8) == rows * per_row * 2 + qo   # K and V
    Lg = W.Layer(num_heads=16, num_kv_heads=1, head_dim=512, k_eq_v=True)
    rows_g = int(lens.sum())
    per_g = (512 + 4) if int8 else 512 * 2
    assert bench.decode_bytes(Lg, lens, int8) == rows_g * per_g + len(lens) * 16 * 512 * 2 * 2   # K only
