"""Host-side multi-GPU plumbing for the indexer: row and sequence sharding.

Query rows of the lightning indexer are independent (each row scores its own
causally visible keys and keeps its own Top-k; "DeepSeek Sparse Attention",
index score equation and the token-selection step), so a prefill chunk splits
into contiguous row blocks, one per GPU, with the keys replicated and no
exchange in the data path; a decode batch splits by sequence.  The row blocks
are balanced by visible pairs, sum over t of (q_offset + t + 1), which is the
work the indexer does per row (2*H*d flops per pair, "DeepSeek DSA FLOPs",
dense indexer cost), not by row count: under a causal mask the last rows of
a chunk see more keys than the first.

The only collectives here are outside the data path: the max-over-ranks
reduction of a timing and an all-gather that brings the disjoint output
blocks together when a caller wants them on every rank.  Everything works
with any torch.distributed backend (NCCL on GPUs, gloo on CPU).
"""

from __future__ import annotations

import torch
import torch.distributed as dist


def balanced_blocks(prefix_work, world: int) -> list[tuple[int, int]]:
    """Split items 0..n-1 into ``world`` contiguous blocks of near-equal work.

    ``prefix_work(i)`` is the total work of items [0, i) (non-decreasing,
    prefix_work(0) == 0); ``n`` is found as the call's ``n`` attribute.
    Block r ends at the item boundary whose prefix is nearest to
    (r+1) / world of the total (a binary search), so every boundary is within
    half an item's work of its target and each block's work within one
    item's work of total / world.  Blocks may be empty when there are fewer
    items than ranks.
    """
    n = prefix_work.n
    total = prefix_work(n)
    bounds = [0]
    for r in range(1, world):
        target = total * r / world
        lo, hi = bounds[-1], n
        while lo < hi:  # first i with prefix_work(i) >= target
            mid = (lo + hi) // 2
            if prefix_work(mid) >= target:
                hi = mid
            else:
                lo = mid + 1
        if lo > bounds[-1] and target - prefix_work(lo - 1) < prefix_work(lo) - target:
            lo -= 1
        bounds.append(lo)
    bounds.append(n)
    return [(bounds[r], bounds[r + 1]) for r in range(world)]


class _CausalPrefix:
    """Visible pairs of rows [0, i): sum over t < i of (q_offset + t + 1)."""

    def __init__(self, T_q: int, q_offset: int):
        self.n, self.q_offset = T_q, q_offset

    def __call__(self, i: int) -> int:
        return i * (self.q_offset + 1) + i * (i - 1) // 2


class _ListPrefix:
    def __init__(self, weights):
        self.n = len(weights)
        self.pre = [0]
        for v in weights:
            self.pre.append(self.pre[-1] + int(v))

    def __call__(self, i: int) -> int:
        return self.pre[i]


def row_shards(T_q: int, q_offset: int, world: int) -> list[tuple[int, int]]:
    """Contiguous query-row blocks [begin, end) of a causal prefill chunk,
    one per rank, balanced by visible pairs.  Rank r calls the prefill
    entry point on rows begin..end-1 with q_offset + begin as its offset and
    the same keys."""
    if T_q < 0 or q_offset < 0 or world < 1:
        raise ValueError("row_shards: T_q >= 0, q_offset >= 0 and world >= 1 are required")
    return balanced_blocks(_CausalPrefix(T_q, q_offset), world)


def sequence_shards(seq_len, world: int) -> list[tuple[int, int]]:
    """Contiguous sequence blocks of a decode batch, balanced by the keys each
    sequence scans (its seq_len)."""
    if world < 1:
        raise ValueError("sequence_shards: world >= 1 is required")
    return balanced_blocks(_ListPrefix([max(0, int(v)) for v in seq_len]), world)


def shard_pairs(T_q: int, q_offset: int, block: tuple[int, int]) -> int:
    """Visible pairs of one row block."""
    p = _CausalPrefix(T_q, q_offset)
    return p(block[1]) - p(block[0])


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of a per-rank scalar (a step time) over all ranks; the
    value itself outside a process group."""
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: int, device=None) -> int:
    """The sum of a per-rank count (pairs processed) over all ranks."""
    if not (dist.is_available() and dist.is_initialized()):
        return int(value)
    t = torch.tensor([int(value)], dtype=torch.int64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return int(t.item())


def gather_row_blocks(local: torch.Tensor, blocks: list[tuple[int, int]]) -> torch.Tensor:
    """All-gather each rank's output rows (block r = rows blocks[r]) into the
    full array on every rank.  ``local`` holds this rank's rows; its trailing
    dimensions are the same on every rank.  Blocks are padded to the largest
    so that one all_gather moves them."""
    if not (dist.is_available() and dist.is_initialized()):
        return local
    world = dist.get_world_size()
    if len(blocks) != world:
        raise ValueError("gather_row_blocks: one block per rank is required")
    rank = dist.get_rank()
    if local.shape[0] != blocks[rank][1] - blocks[rank][0]:
        raise ValueError("gather_row_blocks: local rows do not match this rank's block")
    cap = max(e - b for b, e in blocks)
    pad = local.new_zeros((cap,) + tuple(local.shape[1:]))
    pad[:local.shape[0]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad)
    return torch.cat([parts[r][:e - b] for r, (b, e) in enumerate(blocks)], dim=0)
