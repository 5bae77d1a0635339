"""Host-side sharding of a packed batch across ranks (one process per GPU).

The GDN-2 forward is independent across (sequence, head) units, so a batch
splits across GPUs with no collective on the data path: each rank runs
``chunk_fwd`` on a contiguous range of sequences (balanced by token count)
or on a contiguous range of heads.  These helpers compute the ranges; the
device work on each rank is an ordinary single-GPU call.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple


def sequence_ranges(cu_seqlens: Sequence[int], world: int) -> List[Tuple[int, int]]:
    """Split sequences 0..N-1 into `world` contiguous ranges with token counts as
    even as a greedy left-to-right cut allows.  Ranges may be empty."""
    cu = [int(x) for x in cu_seqlens]
    N, total = len(cu) - 1, cu[-1] - cu[0]
    out, lo = [], 0
    for r in range(world):
        if r == world - 1:
            hi = N
        else:
            target = cu[0] + total * (r + 1) / world
            hi = lo
            while hi < N and abs(cu[hi + 1] - target) <= abs(cu[hi] - target):
                hi += 1
        out.append((lo, hi))
        lo = hi
    return out


def local_problem(cu_seqlens: Sequence[int], rank: int, world: int):
    """This rank's slice: (seq_lo, seq_hi, tok_lo, tok_hi, local cu_seqlens)."""
    cu = [int(x) for x in cu_seqlens]
    lo, hi = sequence_ranges(cu, world)[rank]
    tok_lo, tok_hi = cu[lo], cu[hi]
    return lo, hi, tok_lo, tok_hi, [c - tok_lo for c in cu[lo:hi + 1]]


def head_range(n_heads: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous heads of this rank (head sharding of an equal-length batch)."""
    base, extra = divmod(n_heads, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)
