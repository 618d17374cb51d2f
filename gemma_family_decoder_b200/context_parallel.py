"""Context-parallel prefill: one long prompt over the ranks of a process group.

The model cards give Gemma 4 a 256K context window (KerasFormers "Gemma 4") and
shard training by sequence as well as by batch (Atlas "Gemma 4" summary); a
prompt that long is split over a node's GPUs by query rows.  Rank r owns the
zig-zag token blocks r and 2N-1-r of 2N (gattn_cp_blocks), which gives every
rank the same causal work.  The one exchange step is an all-gather of every
rank's key rows (and value rows, unless the layer's values are its keys) into a
full [B, S, Hkv, D] tensor on each rank, over the process group's backend
(NCCL between GPUs); each owned block then runs as a chunk against the
gathered keys (gattn_prefill_chunk: the block's first token as the prefix
length, no append), so its rows see exactly the keys of a whole-prompt prefill.
Every step of the attention runs in libgattn's kernels; this module only moves
tensors and calls the library.
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence

import torch
import torch.distributed as dist

from .gattn import AttentionLayer, cp_blocks


def gather_rows(blocks: Sequence[torch.Tensor], seq_len: int, group=None) -> torch.Tensor:
    """Every rank's two row blocks [B, len, Hkv, D] (its cp_blocks, in token order)
    assembled into the full [B, seq_len, Hkv, D] tensor on every rank (one all-gather
    of a padded [2, B, Lb, Hkv, D] buffer, Lb the longest block)."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    mine = cp_blocks(seq_len, world, rank)
    for (st, n), t in zip(mine, blocks):
        if t.shape[1] != n:
            raise ValueError(f"block at token {st} has {t.shape[1]} rows, the split gives it {n}")
    B, _, Hkv, D = blocks[0].shape
    Lb = -(-seq_len // (2 * world))
    send = torch.zeros((2, B, Lb, Hkv, D), dtype=blocks[0].dtype, device=blocks[0].device)
    for i, t in enumerate(blocks):
        send[i, :, :t.shape[1]] = t
    recv = [torch.empty_like(send) for _ in range(world)]
    dist.all_gather(recv, send, group=group)
    full = torch.empty((B, seq_len, Hkv, D), dtype=send.dtype, device=send.device)
    for r in range(world):
        for i, (st, n) in enumerate(cp_blocks(seq_len, world, r)):
            full[:, st:st + n] = recv[r][i, :, :n]
    return full


ChunkFn = Callable[[torch.Tensor, torch.Tensor, Optional[torch.Tensor], int], torch.Tensor]


def cp_prefill(layer: AttentionLayer, q_blocks: Sequence[torch.Tensor], k_blocks: Sequence[torch.Tensor],
               v_blocks: Optional[Sequence[torch.Tensor]], seq_len: int, group=None,
               chunk: Optional[ChunkFn] = None):
    """This rank's share of a context-parallel prefill.

    q_blocks / k_blocks / v_blocks: this rank's two blocks of queries [B, len, H, D] and of
    raw keys / values [B, len, Hkv, D] (bf16, positions = token indices), in the order of
    cp_blocks(seq_len, world, rank); v_blocks is None when the layer's values are its keys.
    Returns the two output blocks [B, len, H, D].  `chunk(q_block, k_full, v_full, start)`
    computes one block against the gathered keys; by default it is the library's chunk call.
    """
    k_full = gather_rows(k_blocks, seq_len, group)
    v_full = None if v_blocks is None else gather_rows(v_blocks, seq_len, group)
    if chunk is None:
        def chunk(qb, kf, vf, start):
            pre = torch.full((qb.shape[0],), start, dtype=torch.int32, device=qb.device)
            return layer.prefill_chunk(qb, kf, vf, pre)
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    outs = []
    for (st, n), qb in zip(cp_blocks(seq_len, world, rank), q_blocks):
        outs.append(chunk(qb.contiguous(), k_full, v_full, st) if n > 0 else torch.empty_like(qb))
    return outs
