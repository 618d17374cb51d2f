"""The workspace-free decode entry point against the normal one.

gattn_decode_noalloc is for callers that cannot allocate device memory when
they decode (a fixed, pre-planned memory pool, or no cudaMalloc allowed while
other work runs).  It keeps its split partials in a device array inside the
library instead of a caller workspace.  This test calls it through the C ABI
twice in a row and checks each result against gattn_decode on the same inputs,
within the tolerance the parity tests use.  It sits in a file of its own that
pytest collects last.
"""
import ctypes

import pytest
import torch

import workloads as W
from helpers import MAX_ABS, MEAN_ABS, decode_full_cache, make_layer

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


CASES = [
    # (layer, lengths): the Gemma 4 local and global decode layers, short caches
    ("local_gqa2_w1024", W.GEMMA4_DECODE_LOCAL.layer, [1, 300, 1024, 1500, 2500, 3000]),
    ("global_keqv_d512", W.GEMMA4_DECODE_GLOBAL.layer, [7, 1024, 2049, 3000]),
]


@pytest.mark.parametrize("name,layer,lens", CASES, ids=[c[0] for c in CASES])
def test_noalloc_decode_matches_workspace_decode(name, layer, lens):
    from gemma_family_decoder_b200 import gattn
    L = gattn.lib()
    wl = W.DecodeWorkload(name, layer, len(lens), 1, max(lens), seed=21)
    dq = W.decode_inputs(wl)
    seq_lens = torch.tensor(lens, dtype=torch.int32, device="cuda")
    k, v, _ = decode_full_cache(wl, seq_lens.cpu(), max_len=max(lens) + 3)
    al = make_layer(layer, k.shape[1], dq["w_q"], dq["w_k"])
    q = dq["q"].cuda()
    ref = al.decode(q, k, v, seq_lens)
    torch.cuda.synchronize()
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        st = L.gattn_decode_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                    None if v is None else ctypes.c_void_p(v.data_ptr()),
                                    ctypes.c_void_p(seq_lens.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                    k.shape[0], k.shape[1], ctypes.byref(al.cfg),
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0, L.gattn_last_error()
        torch.cuda.synchronize()
        d = (out.float() - ref.float()).abs()
        assert torch.isfinite(out.float()).all()
        assert d.max().item() <= MAX_ABS and d.mean().item() <= MEAN_ABS


SCRATCH_BYTES = 16 * 1024 * 1024  # the library's scratch array, less two 256-byte roundings below


def test_noalloc_fewer_longer_splits_match_workspace_decode():
    # The Gemma 4 global K=V layer at batch 64: a split slot is 64 * 16 * 514 * 4
    # bytes (2.1 MB), so the 16 MiB array holds 7 slots, while the normal plan
    # for 16384-key caches (2048-key chunks) has 8.  The call must then run 7
    # chunks of 2341 keys (not a multiple of the 128-key tile) and still agree
    # with gattn_decode, twice in a row.
    from gemma_family_decoder_b200 import gattn
    L = gattn.lib()
    layer = W.GEMMA4_DECODE_GLOBAL.layer
    B, max_len = 64, 16384
    per_split = B * layer.num_heads * (layer.head_dim + 2) * 4
    fit = (SCRATCH_BYTES - 512) // per_split
    normal = -(-max_len // 2048)
    assert fit < normal, (fit, normal)             # the reduced plan is the one exercised
    chunk = -(-max_len // fit)
    assert chunk % 128 != 0                        # and its chunks end inside a key tile
    rng = torch.Generator().manual_seed(5)
    lens = torch.randint(1, max_len + 1, (B,), generator=rng, dtype=torch.int32)
    lens[0], lens[1], lens[2] = max_len, chunk, chunk + 1   # a full cache and a chunk's edges
    wl = W.DecodeWorkload("noalloc_reduced", layer, B, 1, max_len, seed=22)
    dq = W.decode_inputs(wl)
    seq_lens = lens.cuda()
    k, v, _ = decode_full_cache(wl, lens, max_len=max_len)
    al = make_layer(layer, max_len, dq["w_q"], dq["w_k"])
    q = dq["q"].cuda()
    ref = al.decode(q, k, v, seq_lens)
    torch.cuda.synchronize()
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        st = L.gattn_decode_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), None,
                                    ctypes.c_void_p(seq_lens.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                    B, max_len, ctypes.byref(al.cfg),
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0, L.gattn_last_error()
        torch.cuda.synchronize()
        d = (out.float() - ref.float()).abs()
        assert torch.isfinite(out.float()).all()
        assert d.max().item() <= MAX_ABS and d.mean().item() <= MEAN_ABS


def test_noalloc_rejects_oversized_batch():
    from gemma_family_decoder_b200 import gattn
    L = gattn.lib()
    layer = W.GEMMA4_DECODE_GLOBAL.layer          # 16 heads x (512 + 2) x 4 B per split and row
    al = make_layer(layer, 64)
    dummy = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    lens = torch.ones(1, dtype=torch.int32, device="cuda")
    p = ctypes.c_void_p(dummy.data_ptr())
    st = L.gattn_decode_noalloc(p, p, None, ctypes.c_void_p(lens.data_ptr()), p, 1024, 64,
                                ctypes.byref(al.cfg), None)
    assert st == 2                                # GATTN_ERR_UNSUPPORTED, nothing launched
    assert b"16 MiB" in L.gattn_last_error()
