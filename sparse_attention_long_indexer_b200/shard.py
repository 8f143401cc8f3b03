"""Query-row sharding of one prefill sequence over the ranks of a process group.

Each rank owns a contiguous range of query rows [r0, r1) of a causal prefill of length L.
The work of row t is its indexer pairs (t + 1 keys, the FP8 contraction and the top-k
epilogue) plus its attention rows (min(t + 1, k) selected rows). The partition balances a
weighted sum of the two, so later ranks get fewer rows.

Each rank holds the key-side cache rows of the tokens it owns: the indexer keys, their
scales and the latent rows. One all-gather assembles the whole caches. The rank then calls
the forward path for its query rows as one chunk, with n_q = r1 - r0 and lengths = r1. By
the header's definition of query positions (pos = len - n_q + i), that call computes exactly
rows r0 .. r1 - 1 of the whole call. Outputs stay sharded.

Host logic only: the exchange is a torch.distributed collective (NCCL on GPUs), and the
forward path runs in the library's kernels.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Sequence

import torch

# Relative cost of one causal (query, key) pair of the indexer and one selected row of the
# attention, from the prefill 128K stage times on one B200: 126.4 ms over 8.59e9 pairs (14.7 ps
# per pair) and 121.9 ms over 2.66e8 rows (458 ps per row).
PAIR_WEIGHT = 1.0
ROW_WEIGHT = 31.0


def cost_prefix(t: int, topk: int, pair_w: float = PAIR_WEIGHT, row_w: float = ROW_WEIGHT) -> float:
    """Work of rows [0, t): sum over u < t of pair_w * (u + 1) + row_w * min(u + 1, topk)."""
    pairs = t * (t + 1) // 2
    if t <= topk:
        rows = t * (t + 1) // 2
    else:
        rows = topk * (topk + 1) // 2 + (t - topk) * topk
    return pair_w * pairs + row_w * rows


def row_partition(L: int, world: int, topk: int, pair_w: float = PAIR_WEIGHT,
                  row_w: float = ROW_WEIGHT) -> List[tuple]:
    """Contiguous row ranges [(r0, r1), ...], one per rank, covering [0, L) in order.

    Boundary j is the first row t at which the work of rows [0, t) reaches j / world of the
    total; ranges may be empty when L < world."""
    if L < 0 or world < 1:
        raise ValueError("L >= 0 and world >= 1 are required")
    total = cost_prefix(L, topk, pair_w, row_w)
    bounds = [0]
    for j in range(1, world):
        target = total * j / world
        lo, hi = bounds[-1], L
        while lo < hi:                                  # first t with cost_prefix(t) >= target
            mid = (lo + hi) // 2
            if cost_prefix(mid, topk, pair_w, row_w) >= target:
                hi = mid
            else:
                lo = mid + 1
        bounds.append(lo)
    bounds.append(L)
    return [(bounds[j], bounds[j + 1]) for j in range(world)]


@dataclass(frozen=True)
class ChunkCall:
    """Arguments of one rank's forward call: its query rows as a chunk of the whole sequence."""
    row0: int        # first query row (its position)
    n_q: int         # rows in the chunk
    length: int      # keys visible to the chunk's last row + 1 = row0 + n_q


def chunk_call(parts: Sequence[tuple], rank: int) -> ChunkCall:
    r0, r1 = parts[rank]
    return ChunkCall(row0=r0, n_q=r1 - r0, length=r1)


def all_gather_rows(local: torch.Tensor, parts: Sequence[tuple], group=None) -> torch.Tensor:
    """Concatenation over ranks of each rank's rows (dim 0), for uneven row counts.

    Every rank pads its rows to the largest range, one all_gather moves the padded blocks,
    and the padding is dropped. ``local`` holds exactly this rank's rows."""
    import torch.distributed as dist
    sizes = [r1 - r0 for (r0, r1) in parts]
    rank = dist.get_rank(group)
    if local.shape[0] != sizes[rank]:
        raise ValueError(f"rank {rank} holds {local.shape[0]} rows, its range has {sizes[rank]}")
    width = max(sizes) if sizes else 0
    padded = local.new_zeros((width,) + tuple(local.shape[1:]))
    padded[: local.shape[0]] = local
    blocks = [torch.empty_like(padded) for _ in parts]
    dist.all_gather(blocks, padded.contiguous(), group=group)
    return torch.cat([b[:n] for b, n in zip(blocks, sizes)], dim=0)
