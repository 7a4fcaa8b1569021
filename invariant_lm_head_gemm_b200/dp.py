"""Data-parallel exchange of the LM-head weight gradient.

Rows (tokens) are independent, so data-parallel ranks need no exchange for
logp, entropy, lse or dHidden.  The one exchange is the sum of the ranks'
local dW.  It is made deterministic -- bitwise the same whatever order the
data arrives in -- by a reduce-scatter done by hand: rank r owns a contiguous
slice of vocab rows, every rank sends its partial slice to the owner with one
all-to-all, and the owner adds the partials in rank order (rlk_sum_ordered).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def slice_rows(V: int, world: int, rank: int):
    """Vocab rows [r0, r1) owned by `rank` (contiguous, near-equal)."""
    per = -(-V // world)
    r0 = min(V, rank * per)
    return r0, min(V, r0 + per)


def reduce_scatter_dw(dW: torch.Tensor, recv: torch.Tensor = None, out: torch.Tensor = None,
                      sum_fn=None, group=None):
    """Deterministic reduce-scatter of dW [V, H] (fp32, contiguous) over the
    ranks of `group`.  Returns (out, r0, r1): out [r1 - r0, H] is the sum over
    ranks, in rank order, of rows r0..r1 of every rank's dW.  `recv` ([world,
    per, H]) and `out` may be preallocated; `sum_fn(parts, out)` adds a list of
    equally shaped tensors in list order (default: the library's
    rlk_sum_ordered)."""
    if sum_fn is None:
        from invariant_lm_head_gemm_b200 import binding
        sum_fn = binding.rlk_sum_ordered
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    V, H = dW.shape
    r0, r1 = slice_rows(V, world, rank)
    rows = r1 - r0
    in_splits = [(b - a) * H for a, b in (slice_rows(V, world, r) for r in range(world))]
    if recv is None:
        recv = torch.empty(world, max(rows, 1), H, dtype=dW.dtype, device=dW.device)
    recv_flat = recv.view(-1)[: world * rows * H]
    dist.all_to_all_single(recv_flat, dW.reshape(-1), [rows * H] * world, in_splits, group=group)
    parts = [recv_flat[k * rows * H:(k + 1) * rows * H] for k in range(world)]
    if out is None:
        out = torch.empty(rows, H, dtype=dW.dtype, device=dW.device)
    if rows > 0:
        sum_fn(parts, out.view(-1)[: rows * H])
    return out, r0, r1
