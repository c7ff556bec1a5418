"""Sequence-sharded prefill: one sequence split into consecutive token ranges, one range
per rank (one process per GPU), with one exchange step.

Every rank
  1. computes its range's final state from a zero start -- the summaries and the scan
     only (``states_only``), no output;
  2. all-gathers the ranges' states (an NCCL all_gather of B*H*(dk*dv + dk) floats per
     rank, 2.1 MB for 32 heads at d = 128);
  3. folds the states of the ranges before its own with the scan page's monoid
     (``lin_attn_combine_states``: P <- gamma^(tokens of range j) P + S_j) -- the
     associative combine of "Log-Depth Chunked Linear-Attention Scan" (Formulas) applied to
     whole ranges, with the decay of "Linear Attention and Retentive Networks ..." (C.
     Chunkwise Recurrent Representation);
  4. runs its range's prefill from that state (``S_init`` / ``Z_init``).

The last rank's final state is the sequence's.  All arithmetic runs in the CUDA library;
this module only moves tensors and calls the collective.  The library functions are
parameters so that the rank logic can be exercised without a GPU.
"""

from __future__ import annotations

from typing import Callable, Sequence

import torch
import torch.distributed as dist

from . import binding as _b
from .ranks import RankInfo


def part_ranges(T: int, world: int, chunk: int = 64) -> list[tuple[int, int]]:
    """(start, length) of each rank's token range: whole chunks, split as evenly as the
    chunk count allows (the last range takes the ragged tail)."""
    n_chunks = -(-T // chunk) if T > 0 else 0
    base, extra = divmod(n_chunks, world)
    ranges, start_chunk = [], 0
    for r in range(world):
        nc = base + (1 if r < extra else 0)
        start = min(T, start_chunk * chunk)
        end = min(T, (start_chunk + nc) * chunk)
        ranges.append((start, end - start))
        start_chunk += nc
    return ranges


def _gather(x: torch.Tensor, info: RankInfo) -> torch.Tensor:
    """Every rank's `x`, stacked in rank order (NCCL on GPUs, gloo on CPU)."""
    if info.world == 1:
        return x.unsqueeze(0).clone()
    parts = [torch.empty_like(x) for _ in range(info.world)]
    dist.all_gather(parts, x.contiguous())
    return torch.stack(parts)


def prefill_sequence_sharded(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                             out: torch.Tensor | None = None, *, info: RankInfo,
                             part_tokens: Sequence[int], gamma=None, normalize: bool = True,
                             prefill: Callable = _b.lin_attn_prefill,
                             combine: Callable = _b.lin_attn_combine_states,
                             gather: Callable = _gather, **kw):
    """This rank's share of a sequence-sharded prefill.

    q, k [B,H,T_r,dk] and v [B,H,T_r,dv] hold this rank's token range; ``part_tokens`` the
    lengths of every rank's range in order.  Returns (out, S_final, Z_final, S_init,
    Z_init): the range's output, the state after its last token and the state before its
    first token.
    """
    if len(part_tokens) != info.world or part_tokens[info.rank] != q.shape[2]:
        raise ValueError("part_tokens must list every rank's range, this rank's matching q")
    _, S_loc, Z_loc = prefill(q, k, v, None, gamma=gamma, normalize=normalize,
                              states_only=True, **kw)
    S_parts = gather(S_loc, info)
    Z_parts = gather(Z_loc, info) if normalize else None
    S_in, Z_in = combine(S_parts, Z_parts, info.rank, list(part_tokens), gamma=gamma)
    out, S_fin, Z_fin = prefill(q, k, v, out, gamma=gamma, normalize=normalize, S_init=S_in,
                                Z_init=Z_in, **kw)
    return out, S_fin, Z_fin, S_in, Z_in
