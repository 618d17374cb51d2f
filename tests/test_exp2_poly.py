"""Error bound of the FMA-pipe 2^a the prefill softmax uses for one weight pair in eight.

`ex2_poly2` (csrc/kernels/common.cuh) splits a = n + f with n = round(a) by the
1.5 * 2^23 rounding trick, evaluates a fitted cubic for 2^f on [-1/2, 1/2] and
adds n to the exponent field.  This test reads the constants from the header and
replays each step in float32 (numpy), then checks the result against 2^a in
float64: relative error below 1e-4 (bf16 weights are rounded to 2^-9 relative)
for every a in [-120, 0], and exactly 0 below -120 (masked entries are -inf).
"""
import re
from pathlib import Path

import numpy as np

HDR = Path(__file__).resolve().parents[1] / "gemma_family_decoder_b200" / "csrc" / "kernels" / "common.cuh"


def _constants():
    src = HDR.read_text()
    body = src[src.index("float2 ex2_poly2(float2 a)"):]
    body = body[:body.index("\n}\n")]
    c = {k: np.float32(float(v)) for k, v in re.findall(r"\b(c[0-3]) = ([0-9.eE+-]+)f", body)}
    k_round = np.float32(float(re.search(r"kRound = ([0-9.]+)f", body).group(1)))
    return c, k_round


def _ex2_poly(a):
    c, k_round = _constants()
    a = np.asarray(a, dtype=np.float32)
    zero = a < np.float32(-120.0)
    a = np.where(zero, np.float32(-120.0), a).astype(np.float32)
    t = (a + k_round).astype(np.float32)
    r = (t - k_round).astype(np.float32)
    f = (a - r).astype(np.float32)
    p = (c["c3"] * f + c["c2"]).astype(np.float32)
    p = (p * f + c["c1"]).astype(np.float32)
    p = (p * f + c["c0"]).astype(np.float32)
    bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    out = bits.astype(np.uint32).view(np.float32)
    return np.where(zero, np.float32(0.0), out)


def test_constants_present():
    c, k_round = _constants()
    assert set(c) == {"c0", "c1", "c2", "c3"}
    assert k_round == np.float32(1.5 * 2 ** 23)


def test_relative_error_bound():
    a = np.concatenate([np.linspace(-120.0, 0.0, 400001), -np.random.default_rng(0).random(100000) * 120.0])
    a = a.astype(np.float32)
    got = _ex2_poly(a).astype(np.float64)
    ref = np.exp2(a.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1e-4, rel.max()


def test_exact_on_integers_and_zero_below_range():
    # f = 0: the result is c0 * 2^n, within the bound of 2^n
    n = np.arange(-120, 1, dtype=np.float32)
    assert np.all(np.abs(_ex2_poly(n) / np.exp2(n.astype(np.float64)) - 1.0) < 1e-4)
    below = np.array([-120.5, -200.0, -np.inf], dtype=np.float32)
    assert np.all(_ex2_poly(below) == 0.0)
