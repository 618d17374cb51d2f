"""Context-parallel prefill on CPU ranks (gloo): the split, the key all-gather and
the per-block chunk reproduce the whole-prompt layer.

The split (gattn_cp_blocks, through the C ABI; host only) must cover the prompt
once, give rank r the zig-zag blocks r and 2N-1-r, and balance the causal work.
Two and three gloo ranks then run gemma_family_decoder_b200.context_parallel on
a small Gemma-4-shaped layer (head_dim 512, K=V, partial RoPE, plain-weight
QK-norm; and one layer with separate values and a window): each gathers the
keys (and values) over the process group and computes its blocks with the
float64 oracle's chunk function standing in for the GPU kernel; the blocks put
together equal the oracle's whole-prompt prefill to 1e-9.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("S", [0, 1, 5, 64, 255, 300, 32768])
@pytest.mark.parametrize("N", [1, 2, 3, 4, 8])
def test_cp_blocks_cover_the_prompt_once_and_balance(S, N):
    from gemma_family_decoder_b200.gattn import cp_blocks
    nb = 2 * N
    # the 2N blocks, as evenly as possible, the longer ones first
    lens = [S // nb + (1 if i < S % nb else 0) for i in range(nb)]
    starts = [sum(lens[:i]) for i in range(nb)]
    seen = np.zeros(S, dtype=int)
    work = []
    for r in range(N):
        got = cp_blocks(S, N, r)
        assert got == [(starts[r], lens[r]), (starts[nb - 1 - r], lens[nb - 1 - r])]
        w = 0
        for st, n in got:
            seen[st:st + n] += 1
            w += sum(i + 1 for i in range(st, st + n))   # visible keys of each query row
        work.append(w)
    assert (seen == 1).all()
    if S % nb == 0:
        assert len(set(work)) == 1                        # exactly equal causal work
    else:
        assert max(work) - min(work) <= 2 * S             # within one row's keys per extra token


def test_cp_blocks_rejects_bad_arguments():
    from gemma_family_decoder_b200.gattn import GattnError, cp_blocks
    for args in ((10, 0, 0), (10, 2, 2), (10, 2, -1), (-1, 2, 0)):
        with pytest.raises(GattnError):
            cp_blocks(*args)


def _rank_main(rank, world, port, case, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch.distributed as dist

    import oracle as O
    from gemma_family_decoder_b200.context_parallel import cp_prefill
    from gemma_family_decoder_b200.gattn import cp_blocks
    from helpers import small_prefill_inputs
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world)
        layer, S, gm = case
        d = small_prefill_inputs(layer, 1, S, seed=77, gain_mean=gm)
        mine = cp_blocks(S, world, rank)
        qb = [d["q"][:, st:st + n] for st, n in mine]
        kb = [d["k"][:, st:st + n] for st, n in mine]
        vb = None if d["v"] is None else [d["v"][:, st:st + n] for st, n in mine]

        def oracle_chunk(q_blk, k_full, v_full, start):
            # stands in for the library's chunk call on this CPU-only host
            pre = torch.full((q_blk.shape[0],), start, dtype=torch.int32)
            return torch.from_numpy(O.attention_prefill_chunk(q_blk, k_full, v_full, pre, layer,
                                                              w_q=d["w_q"], w_k=d["w_k"]))

        outs = cp_prefill(None, qb, kb, vb, S, chunk=oracle_chunk)
        out_q.put((rank, [(st, o.numpy()) for (st, _), o in zip(mine, outs)]))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def _run_ranks(world, case):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0] * world, codes
    return got


@pytest.mark.parametrize("world,S,over", [
    (2, 300, {}),                                                  # Gemma-4 global: K=V, partial RoPE, w-norm
    (3, 301, {}),
    (2, 260, dict(k_eq_v=False, window=90, softcap=30.0, qk_norm=0, rotary_fraction=1.0, rope_theta=1e4)),
])
def test_cp_prefill_blocks_equal_the_whole_prompt(world, S, over):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle as O
    import workloads as W
    from helpers import small_prefill_inputs
    base = dict(head_dim=512, num_heads=4, num_kv_heads=1, k_eq_v=True, rotary_fraction=0.25, rope_theta=1e6,
                qk_norm=W.NORM_W, scalar=512.0)
    layer = W.Layer(**{**base, **over})
    gm = 1.0 if layer.qk_norm == W.NORM_W else 0.0
    got = _run_ranks(world, (layer, S, gm))
    d = small_prefill_inputs(layer, 1, S, seed=77, gain_mean=gm)
    ref = O.attention_prefill(d["q"], d["k"], d["v"], d["positions"], layer, w_q=d["w_q"], w_k=d["w_k"])
    full = np.full(ref.shape, np.nan)
    for _, blocks in got:
        for st, o in blocks:
            full[:, st:st + o.shape[1]] = o
    assert np.isfinite(full).all()                                  # every row came from exactly one rank
    assert np.max(np.abs(full - ref)) < 1e-9
