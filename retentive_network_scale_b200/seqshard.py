"""Chunkwise retention of one long sequence split over several ranks, one
segment of consecutive rows per rank.

"Retentive Network" paper summary, section 2.1, chunkwise form (3): a block
of rows that starts from state R leaves gamma^n R + U, where U (the state
the block leaves from a zero start) depends on the block alone.  Segments
are such blocks, so a rank needs only the other segments' U to start its own
segment from the exact state:

1. U of the own segment (``ret_segment_state``: a streaming pass over K and
   one batched GEMM; no output rows are computed),
2. an all-gather of the U over the ranks (NCCL through ``torch.distributed``
   on GPUs; the one exchange of the path),
3. the state entering the own segment (``ret_state_scan``),
4. the segment's outputs (``ret_chunkwise`` from that state, at the
   segment's absolute positions, with the fused GroupNorm and gate if asked).

Every rank holds only its own rows of Q, K, V (and G).  The rank that holds
the last segment gets the state after the whole sequence in ``state_out``.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Optional, Sequence

import torch

from . import retention as R


def segment_lengths(L: int, parts: int, multiple: int = 128) -> list:
    """Lengths of `parts` consecutive segments covering L rows: as equal as
    possible, every boundary on a multiple of `multiple` while that leaves
    each segment at least one row; the remainder goes to the last."""
    if parts < 1 or L < parts:
        raise ValueError(f"cannot cut {L} rows into {parts} non-empty segments")
    base = (L // parts) // multiple * multiple
    if base == 0:
        base = L // parts
    lens = [base] * (parts - 1)
    lens.append(L - base * (parts - 1))
    return lens


@dataclass
class SegmentOps:
    """The three computations of a rank.  The defaults are the library's
    CUDA entry points; tests substitute others to check the exchange logic
    without a GPU."""
    segment_state: Callable = R.ret_segment_state
    state_scan: Callable = R.ret_state_scan
    chunkwise: Callable = R.ret_chunkwise


def all_gather_states(U: torch.Tensor, group=None) -> torch.Tensor:
    """[world][...] stack of every rank's U, in rank order."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    parts = [torch.empty_like(U) for _ in range(world)]
    dist.all_gather(parts, U.contiguous(), group=group)
    return torch.stack(parts)


def chunkwise_sequence_sharded(Q, K, V, gamma, chunk, seg_lens: Sequence[int], rank: int, *,
                               O=None, G=None, Y=None, state_in=None, state_out=None,
                               gn_eps=1e-5, rotate=False, theta_base=10000.0, pos_offset=0,
                               group=None, gather: Optional[Callable] = None,
                               ops: Optional[SegmentOps] = None, stream=None):
    """Outputs of segment `rank` of a sequence cut into ``seg_lens``.

    Q, K [B][H][seg_lens[rank]][d_k] and V [B][H][seg_lens[rank]][d_v] hold
    this rank's rows (G [B][seg_lens[rank]][H*d_v] likewise); ``state_in``
    is the state before the first segment, the same on every rank (or
    None); ``pos_offset`` is the absolute position of the first segment's
    first row.  ``gather`` replaces the all-gather over ``group`` (it
    receives this rank's U and returns all of them in rank order).  Returns
    (O, Y, state_out) like ``ret_chunkwise``; state_out is the state after
    this segment, which on the last rank is that after the whole sequence.
    """
    ops = ops or SegmentOps()
    seg_lens = [int(n) for n in seg_lens]
    if not 0 <= rank < len(seg_lens):
        raise ValueError(f"rank {rank} outside 0..{len(seg_lens) - 1}")
    if Q.shape[2] != seg_lens[rank]:
        raise ValueError(f"Q holds {Q.shape[2]} rows, segment {rank} has {seg_lens[rank]}")
    start = pos_offset + sum(seg_lens[:rank])
    kw = dict(rotate=rotate, theta_base=theta_base)
    U = ops.segment_state(K, V, gamma, pos_offset=start, stream=stream, **kw)
    U_all = gather(U) if gather is not None else all_gather_states(U, group)
    if U_all.shape[0] != len(seg_lens):
        raise ValueError(f"{U_all.shape[0]} states gathered for {len(seg_lens)} segments")
    Rin = ops.state_scan(U_all, seg_lens, rank, gamma, state_in=state_in, stream=stream)
    return ops.chunkwise(Q, K, V, gamma, chunk, O=O, G=G, Y=Y, state_in=Rin,
                         state_out=state_out, gn_eps=gn_eps, pos_offset=start, stream=stream, **kw)
