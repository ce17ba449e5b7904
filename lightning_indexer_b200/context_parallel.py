"""Context-parallel DSA prefill of one long sequence over the ranks of a process group.

A sequence too long for one GPU's time budget is split by query rows: with N ranks the L
positions form 2N equal blocks and rank r owns blocks r and 2N-1-r (an early and a late
block, so every rank has about the same causal work).  Each rank holds the query-side
inputs (q_idx, w, Q) and the key-side inputs (k_idx, K, V) of its own positions.  The one
exchange is an all-gather of the key side, after which every rank holds the whole
sequence's keys and computes its rows with no further communication: a block of rows
[a, b) is a query chunk whose rows see keys 0 .. b-1 with bottom-right alignment (row i of
the chunk is position a + i), so the library's calls run on it unchanged.

Only the host-side orchestration lives here: the partition, the all-gather (NCCL over
NVLink on GPUs; any torch.distributed backend works) and the per-block calls.  The
per-block computation is a callable, the library's own `prefill_block` by default.
"""
from typing import Callable, List, Optional, Sequence, Tuple

import torch


def zigzag_blocks(L: int, world: int) -> List[Tuple[int, int]]:
    """The 2 * world position blocks [a, b) of a length-L sequence, in position order."""
    n = 2 * world
    bounds = [(L * j) // n for j in range(n + 1)]
    return [(bounds[j], bounds[j + 1]) for j in range(n)]


def rank_blocks(L: int, world: int, rank: int) -> List[Tuple[int, int]]:
    """The position blocks rank `rank` owns: block `rank` and block 2 * world - 1 - rank."""
    blocks = zigzag_blocks(L, world)
    return [blocks[rank], blocks[2 * world - 1 - rank]]


def local_rows(L: int, world: int, rank: int) -> torch.Tensor:
    """The sequence positions of this rank's rows, in the order its local tensors hold them."""
    return torch.cat([torch.arange(a, b) for a, b in rank_blocks(L, world, rank)])


def gather_keys(local: Sequence[torch.Tensor], L: int, world: int, rank: int, group=None) -> List[torch.Tensor]:
    """All-gathers key-side tensors whose first dimension runs over this rank's positions and
    returns them whole, in position order.

    Every rank holds the same number of rows only when 2 * world divides L; the blocks are
    padded to the longest block for the collective and trimmed afterwards.
    """
    import torch.distributed as dist
    blocks = zigzag_blocks(L, world)
    pad = max(b - a for a, b in blocks)
    out = []
    for t in local:
        mine = rank_blocks(L, world, rank)
        rest = tuple(t.shape[1:])
        buf = torch.zeros((2 * pad,) + rest, dtype=t.dtype, device=t.device)
        n0 = mine[0][1] - mine[0][0]
        buf[:n0] = t[:n0]
        buf[pad:pad + (t.shape[0] - n0)] = t[n0:]
        parts = [torch.empty_like(buf) for _ in range(world)]
        dist.all_gather(parts, buf, group=group)
        full = torch.empty((L,) + rest, dtype=t.dtype, device=t.device)
        for r, part in enumerate(parts):
            for j, (a, b) in enumerate(rank_blocks(L, world, r)):
                full[a:b] = part[j * pad:j * pad + (b - a)]
        out.append(full)
    return out


def prefill_block(q_idx, w, Q, k_idx_full, K_full, V_full, a: int, b: int, k: int, chunk_rows: int = 8192,
                  scale: Optional[float] = None):
    """DSA prefill of the query rows at positions [a, b) of one sequence whose keys up to b
    are in the *_full tensors (q_idx, w, Q hold just these rows).  Returns (indices, O, lse)
    with sequence positions in the indices."""
    from . import prefill
    dev = Q.device
    cu_q = torch.tensor([0, b - a], dtype=torch.int32, device=dev)
    cu_k = torch.tensor([0, b], dtype=torch.int32, device=dev)
    return prefill(q_idx, k_idx_full[:b], w, Q, K_full[:b], V_full[:b], cu_q, cu_k, b - a, b, k,
                   chunk_rows=min(chunk_rows, b - a), scale=scale)


def prefill_context_parallel(q_idx, k_idx, w, Q, K, V, L: int, k: int, group=None,
                             block_fn: Optional[Callable] = None, chunk_rows: int = 8192):
    """Context-parallel prefill: this rank's (indices, O, lse), rows in local_rows() order.

    q_idx, w, Q, k_idx, K, V hold this rank's positions (local_rows order).  The key side
    is all-gathered once; each of the rank's two blocks then runs
    block_fn(q_idx_block, w_block, Q_block, k_idx_full, K_full, V_full, a, b) (default:
    prefill_block, the library's kernels).
    """
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    k_idx_full, K_full, V_full = gather_keys([k_idx, K, V], L, world, rank, group)
    fn = block_fn or (lambda *args: prefill_block(*args, k, chunk_rows=chunk_rows))
    outs = []
    off = 0
    for a, b in rank_blocks(L, world, rank):
        n = b - a
        outs.append(fn(q_idx[off:off + n], w[off:off + n], Q[off:off + n], k_idx_full, K_full, V_full, a, b))
        off += n
    return tuple(torch.cat([o[i] for o in outs]) for i in range(3))
