"""Sequence sharding for running the fused ShortConv K/V step on several GPUs.

The step has no cross-sequence dependency: a sequence's outputs depend only
on its own rows, its own conv_state and the shared taps/gammas.  So a batch
is split across ranks by whole sequences, each rank owning its sequences'
state rows and cache pages, and no collective is needed on the data path
(one process per GPU; NCCL is used only for barriers and for taking the
slowest rank's time).

partition_sequences() cuts the packed sequence list into `world` contiguous
groups with near-equal token counts, so every rank gets a contiguous slice of
k/v rows and of slot_mapping.
"""
from typing import List, Sequence


def partition_sequences(lengths: Sequence[int], world: int) -> List[range]:
    """Split sequences 0..S-1 into `world` contiguous ranges whose token
    totals are as even as whole sequences allow: rank r takes the sequences
    whose token prefix midpoint falls in [r*T/world, (r+1)*T/world)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    S = len(lengths)
    total = sum(int(x) for x in lengths)
    bounds = [0] * (world + 1)
    bounds[world] = S
    if total == 0:
        for r in range(world + 1):
            bounds[r] = min(S, (S * r) // world)
        return [range(bounds[r], bounds[r + 1]) for r in range(world)]
    r, acc = 1, 0
    for i, L in enumerate(lengths):
        mid2 = 2 * acc + int(L)  # twice the midpoint, to stay in integers
        while r < world and mid2 >= 2 * total * r // world:
            bounds[r] = i
            r += 1
        acc += int(L)
    while r < world:
        bounds[r] = S
        r += 1
    return [range(bounds[r], bounds[r + 1]) for r in range(world)]


def token_range(lengths: Sequence[int], seqs: range):
    """[first, last) packed-token rows of a contiguous sequence range."""
    start = sum(int(x) for x in lengths[:seqs.start])
    stop = start + sum(int(x) for x in lengths[seqs.start:seqs.stop])
    return start, stop


def local_view(batch, seqs: range):
    """The part of a packed workloads.Batch that one rank owns: its rows of
    k/v and slot_mapping, a rebased cu_seqlens, and state indices that point
    into the shared pool (identity indices become explicit)."""
    import torch
    from .workloads import Batch
    lengths = (batch.cu_seqlens[1:] - batch.cu_seqlens[:-1]).tolist()
    a, b = token_range(lengths, seqs)
    cu = batch.cu_seqlens[seqs.start:seqs.stop + 1] - batch.cu_seqlens[seqs.start]
    if batch.state_indices is None:
        si = torch.arange(seqs.start, seqs.stop, dtype=torch.int32)
    else:
        si = batch.state_indices[seqs.start:seqs.stop].clone()
    return Batch(W=batch.W, Hkv=batch.Hkv, D=batch.D, eps=batch.eps, k=batch.k[a:b],
                 v=batch.v[a:b], cu_seqlens=cu.to(torch.int32).contiguous(),
                 conv_w_k=batch.conv_w_k, conv_w_v=batch.conv_w_v,
                 gamma_k=batch.gamma_k, gamma_v=batch.gamma_v,
                 conv_state=batch.conv_state, slot_mapping=batch.slot_mapping[a:b],
                 num_pages=batch.num_pages, page_size=batch.page_size,
                 state_indices=si, meta=dict(batch.meta, rows=(a, b), seqs=(seqs.start, seqs.stop)))
