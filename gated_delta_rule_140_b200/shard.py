"""Data-parallel sharding of a packed batch across ranks.

The gated delta rule's (sequence, head) chains are independent, so a batch
shards across GPUs with no communication on the data path: each rank runs
gdn_chunk_fwd on its own sequences.  ``shard_sequences`` balances the ranks by
token count (longest sequence first onto the least-loaded rank), and
``local_batch`` packs one rank's sequences into a contiguous varlen batch.
"""
from __future__ import annotations

import heapq

import torch


def shard_sequences(lengths, world: int) -> list[list[int]]:
    """Assign sequence indices to ``world`` ranks, balancing total tokens.

    Greedy longest-processing-time: sequences in decreasing length go to the
    rank with the fewest tokens so far (ties by rank id).  Each rank's list is
    returned in increasing sequence order.  Deterministic."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(lengths)), key=lambda i: (-int(lengths[i]), i))
    heap = [(0, r) for r in range(world)]
    out = [[] for _ in range(world)]
    for i in order:
        load, r = heapq.heappop(heap)
        out[r].append(i)
        heapq.heappush(heap, (load + int(lengths[i]), r))
    return [sorted(x) for x in out]


def local_batch(x: dict, seqs: list[int]) -> dict:
    """Pack the sequences ``seqs`` of a varlen batch ``x`` (q, k, v, log_alpha,
    beta with B = 1 and int32 cu_seqlens; optional initial_state) into a new
    contiguous varlen batch.  Works on CPU or CUDA tensors."""
    cu = x["cu_seqlens"].tolist()
    parts = {n: [] for n in ("q", "k", "v", "log_alpha", "beta")}
    lens = []
    for i in seqs:
        s, e = cu[i], cu[i + 1]
        lens.append(e - s)
        for n in parts:
            parts[n].append(x[n][:, s:e])
    out = {n: (torch.cat(p, dim=1) if p else x[n][:, :0]) for n, p in parts.items()}
    new_cu = torch.zeros(len(seqs) + 1, dtype=torch.int32)
    if lens:
        new_cu[1:] = torch.cumsum(torch.tensor(lens), 0).to(torch.int32)
    out["cu_seqlens"] = new_cu.to(x["cu_seqlens"].device)
    s0 = x.get("initial_state")
    out["initial_state"] = None if s0 is None else s0[seqs]
    return out
