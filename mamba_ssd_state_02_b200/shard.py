"""Data-parallel prefill over several GPUs: each rank takes whole sequences of a packed
batch. Sequences are independent in the SSD scan (each starts from its own initial state),
so the ranks exchange nothing while they compute; only the caller's gather of the outputs,
if it wants them in one place, crosses devices.

`shard_sequences` balances tokens: sequences are taken longest first and each goes to the
rank with the fewest tokens so far (longest-processing-time-first scheduling). A rank's
sequences keep their original order. `local_batch` gives one rank's packed token rows and
its own `cu_seqlens`; `take_rows` gathers those rows of a `[T, ...]` tensor.
"""
from __future__ import annotations

import torch


def shard_sequences(seqlens: list[int], world: int) -> list[list[int]]:
    """Sequence indices per rank (each sequence on exactly one rank)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(seqlens)), key=lambda i: (-int(seqlens[i]), i))
    load = [0] * world
    ranks: list[list[int]] = [[] for _ in range(world)]
    for i in order:
        r = min(range(world), key=lambda k: (load[k], k))
        ranks[r].append(i)
        load[r] += int(seqlens[i])
    return [sorted(ix) for ix in ranks]


def local_batch(cu_seqlens: list[int], indices: list[int]) -> tuple[list[tuple[int, int]], list[int]]:
    """Token row ranges [start, end) of the given sequences in the packed batch, and the
    `cu_seqlens` of the rank's own packed batch of them."""
    spans = [(int(cu_seqlens[i]), int(cu_seqlens[i + 1])) for i in indices]
    cu = [0]
    for a, b in spans:
        cu.append(cu[-1] + (b - a))
    return spans, cu


def take_rows(t: torch.Tensor, spans: list[tuple[int, int]]) -> torch.Tensor:
    """Rows [a, b) of t for each span, concatenated in order (a new contiguous tensor)."""
    if not spans:
        return t[:0].clone()
    return torch.cat([t[a:b] for a, b in spans], dim=0)
