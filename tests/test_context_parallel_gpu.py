"""Context-parallel prefill through the library's chunk kernel, against the oracle.

Every rank of a context-parallel prefill (gemma_family_decoder_b200.context_parallel)
runs its two zig-zag blocks as chunks (gattn_prefill_chunk) against the gathered
keys.  Here one GPU runs the per-rank work of 2 and 4 ranks one after the other,
each rank's blocks against the full key tensor the all-gather would give it, and
the blocks put together must match the float64 oracle's whole-prompt prefill
(max-abs 2e-2, mean-abs 2e-3).  cp_prefill itself runs on a one-rank NCCL group.
The layer is Gemma-4-shaped (head_dim 512, K=V, partial RoPE, plain-weight
QK-norm; KerasFormers "Gemma 4", What changed).
"""
import os
import socket

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from helpers import assert_close, make_layer, small_prefill_inputs, to_dev

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

G4 = W.Layer(head_dim=512, num_heads=4, num_kv_heads=1, k_eq_v=True, rotary_fraction=0.25, rope_theta=1e6,
             qk_norm=W.NORM_W, scalar=512.0)


@pytest.mark.parametrize("world,S", [(2, 700), (4, 1031)])
def test_rank_blocks_through_chunk_kernel_match_oracle(world, S):
    from gemma_family_decoder_b200.gattn import cp_blocks
    d = small_prefill_inputs(G4, 1, S, seed=91, gain_mean=1.0)
    L = make_layer(G4, S, d["w_q"], d["w_k"])
    dv = to_dev(d)
    out = torch.full_like(dv["q"], float("nan"))
    for r in range(world):
        for st, n in cp_blocks(S, world, r):
            if n == 0:
                continue
            pre = torch.tensor([st], dtype=torch.int32, device="cuda")
            out[:, st:st + n] = L.prefill_chunk(dv["q"][:, st:st + n].contiguous(), dv["k"], None, pre)
    torch.cuda.synchronize()
    ref = O.attention_prefill(d["q"], d["k"], None, d["positions"], G4, w_q=d["w_q"], w_k=d["w_k"])
    assert_close(out, ref, f"{world} ranks")


def test_cp_prefill_on_a_one_rank_nccl_group():
    import torch.distributed as dist
    from gemma_family_decoder_b200.context_parallel import cp_prefill
    from gemma_family_decoder_b200.gattn import cp_blocks
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    S = 513
    d = small_prefill_inputs(G4, 1, S, seed=92, gain_mean=1.0)
    L = make_layer(G4, S, d["w_q"], d["w_k"])
    dv = to_dev(d)
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        mine = cp_blocks(S, 1, 0)
        outs = cp_prefill(L, [dv["q"][:, st:st + n] for st, n in mine], [dv["k"][:, st:st + n] for st, n in mine],
                          None, S)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ref = O.attention_prefill(d["q"], d["k"], None, d["positions"], G4, w_q=d["w_q"], w_k=d["w_k"])
    got = np.concatenate([o.float().cpu().numpy() for o in outs], axis=1)
    order = np.concatenate([np.arange(st, st + n) for st, n in mine])
    assert_close(torch.from_numpy(got), ref[:, order], "one-rank cp_prefill")
