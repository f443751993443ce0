"""Data-parallel sharding of a jagged HSTU batch across ranks.

Sequences are independent in the forward (no term couples two users), so a
global batch splits by whole sequences with no data-path collective.  The
backward's only shared state is the parameter gradients -- the rab tables and
the LayerNorm affine -- which data parallelism sums across ranks with one
small all-reduce.

Balance: MTGR's training system sizes each GPU's batch by its total token count
(MTGR deep-dive, section 3, contribution 3).  For attention the cost grows as
L^2, so the greedy longest-first assignment below balances sum(L^2) and
breaks ties by tokens.
"""
from __future__ import annotations

from typing import Dict, List, Sequence

import numpy as np
import torch

PARAM_GRADS = ("d_rab_pos", "d_rab_time", "d_gamma", "d_beta")


def partition_sequences(lengths: Sequence[int], world: int) -> List[List[int]]:
    """Assign sequence indices to ranks: longest first, each to the least-loaded rank."""
    L = np.asarray(lengths, dtype=np.int64)
    order = sorted(range(len(L)), key=lambda b: (-int(L[b]) * int(L[b]), b))
    cost = [0] * world
    tokens = [0] * world
    parts: List[List[int]] = [[] for _ in range(world)]
    for b in order:
        r = min(range(world), key=lambda k: (cost[k], tokens[k], k))
        parts[r].append(b)
        cost[r] += int(L[b]) * int(L[b])
        tokens[r] += int(L[b])
    return [sorted(p) for p in parts]


def rank_sequences(lengths: Sequence[int], world: int, rank: int) -> List[int]:
    """The sequences of a global batch that rank `rank` of `world` processes (the
    cost-balanced partition above; every rank computes the same partition)."""
    return partition_sequences(lengths, world)[rank]


def shard_rows(offsets: np.ndarray, seqs: Sequence[int]):
    """(new offsets, global row indices) of the listed sequences, in order."""
    off = np.asarray(offsets, dtype=np.int64)
    lens = np.array([off[b + 1] - off[b] for b in seqs], dtype=np.int64)
    new = np.zeros(len(seqs) + 1, dtype=np.int64)
    new[1:] = np.cumsum(lens)
    rows = np.concatenate([np.arange(off[b], off[b + 1]) for b in seqs]) if len(seqs) else np.zeros(0, np.int64)
    return new.astype(np.int32), rows


def bin_sequences(bin_seq_start, rank: int) -> List[int]:
    """The sequences of token-balanced bin `rank` (contiguous: [start[rank], start[rank + 1]))."""
    a, z = int(bin_seq_start[rank]), int(bin_seq_start[rank + 1])
    return list(range(a, z))


def allreduce_param_grads(grads: Dict[str, torch.Tensor], group=None, weight: float = 1.0) -> None:
    """Sum weight * (parameter gradients) over the process group in place (one flat all-reduce).
    With token-balanced bins, each rank's per-sample mean gradient carries weight = its samples /
    all samples (MTGR's re-weighted aggregation), so the sum is the mean over the whole batch."""
    import torch.distributed as dist
    ts = [grads[k] for k in PARAM_GRADS]
    flat = torch.cat([t.reshape(-1) for t in ts])
    if weight != 1.0:
        flat.mul_(weight)
    dist.all_reduce(flat, group=group)
    o = 0
    for t in ts:
        n = t.numel()
        t.copy_(flat[o:o + n].view_as(t))
        o += n
