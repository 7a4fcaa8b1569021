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


# ---------------------------------------------------------------------------
# The same exchange overlapped with the backward.  The backward finishes its
# vocab chunks (rlk_bwd_chunk_width(V) rows each) roughly in ascending order
# and can publish each one (rlk_linear_logp_bwd_signal).  The exchange then
# runs one group of consecutive chunks at a time on a second stream, each
# group's collective waiting on the device for its chunks' completion words, so
# the transfer of finished rows overlaps the computation of later ones.  Every
# element is still the rank-ordered sum; only the row ownership differs: in
# every group each rank owns the near-equal contiguous part slice_rows gives it
# of the group's rows.
# ---------------------------------------------------------------------------


def group_rows(V: int, chunk: int, group_chunks: int):
    """(g0, g1, c0, c1) per group: rows [g0, g1) = chunks [c0, c1)."""
    n = -(-V // chunk)
    out = []
    for c0 in range(0, n, group_chunks):
        c1 = min(n, c0 + group_chunks)
        out.append((c0 * chunk, min(V, c1 * chunk), c0, c1))
    return out


def owned_pieces(V: int, chunk: int, group_chunks: int, world: int, rank: int):
    """Rows [r0, r1) that `rank` owns in each group, in group order."""
    pieces = []
    for g0, g1, _, _ in group_rows(V, chunk, group_chunks):
        a, b = slice_rows(g1 - g0, world, rank)
        pieces.append((g0 + a, g0 + b))
    return pieces


def reduce_scatter_dw_overlapped(dW: torch.Tensor, chunk: int, chunk_done=None, seq: int = 0,
                                 group_chunks: int = 4, stream=None, recv=None, out=None,
                                 sum_fn=None, wait_fn=None, group=None):
    """Deterministic reduce-scatter of dW [V, H] one group of vocab chunks at a
    time.  Before a group's collective, `stream` waits (on the device) until the
    completion words chunk_done[c] of the group's chunks hold seq or more
    (skipped when chunk_done is None).  Returns (out, pieces): out holds this
    rank's rows of every group in group order, pieces their (r0, r1) in dW."""
    import contextlib
    if sum_fn is None or wait_fn is None:
        from invariant_lm_head_gemm_b200 import binding
        sum_fn = sum_fn or binding.rlk_sum_ordered
        wait_fn = wait_fn or binding.rlk_stream_wait_chunk
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    V, H = dW.shape
    groups = group_rows(V, chunk, group_chunks)
    pieces = owned_pieces(V, chunk, group_chunks, world, rank)
    total = sum(b - a for a, b in pieces)
    most = max(b - a for a, b in pieces)
    if out is None:
        out = torch.empty(max(total, 1), H, dtype=dW.dtype, device=dW.device)
    if recv is None:
        recv = torch.empty(world * max(most, 1) * H, dtype=dW.dtype, device=dW.device)
    ctx = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
    with ctx:
        off = 0
        for (g0, g1, c0, c1), (p0, p1) in zip(groups, pieces):
            if chunk_done is not None:
                for c in range(c0, c1):
                    wait_fn(chunk_done[c:c + 1], seq, stream)
            rows = p1 - p0
            in_splits = [(b - a) * H for a, b in (slice_rows(g1 - g0, world, r)
                                                  for r in range(world))]
            rv = recv[: world * rows * H]
            dist.all_to_all_single(rv, dW[g0:g1].reshape(-1), [rows * H] * world, in_splits,
                                   group=group)
            if rows > 0:
                sum_fn([rv[k * rows * H:(k + 1) * rows * H] for k in range(world)],
                       out.view(-1)[off * H:(off + rows) * H])
            off += rows
    return out, pieces
