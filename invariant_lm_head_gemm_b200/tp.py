"""Vocab-parallel (tensor-parallel) linear-logp, forward and backward.

Each rank holds a contiguous shard of the LM head W on the grid of
shard_alignment(V) rows: a multiple of both the forward's split width (512)
and the backward's chunk width (8192 for large vocabularies).  Splits and
chunks then lie wholly in one shard, every rank computes exactly the split
triples, dlogits, dW rows and per-chunk dHidden products that the single-GPU
path computes for its rows, and the fixed-order merges give logp, entropy,
lse, dHidden and dW bit for bit equal to one GPU's, for any number of ranks.

Exchange per step: forward, three all-gathers of [T, Gs] fp32 split triples
and one all-reduce of the [T] target logits (one non-zero term per row);
backward, one all-to-all of the per-chunk dHidden products (each rank
receives its row slice of every chunk) and one all-gather of the bf16
dHidden row slices.  dW stays sharded like W.
"""
from __future__ import annotations

import math

import torch
import torch.distributed as dist

from invariant_lm_head_gemm_b200 import binding


def _cdiv(a: int, b: int) -> int:
    return -(-a // b)


def shard_alignment(V: int, split: int = 512, chunk: int = None) -> int:
    """Row grid of the shards: whole forward splits and backward chunks."""
    if chunk is None:
        chunk = binding.bwd_chunk_width(V)
    return split * chunk // math.gcd(split, chunk)


def shard_rows(V: int, world: int, rank: int, align: int):
    """Vocab rows [v0, v1) of `rank`: equal shards of whole `align`-row blocks
    (the last non-empty shard takes what is left; later ones are empty)."""
    per = _cdiv(_cdiv(V, world), align) * align
    v0 = min(V, rank * per)
    return v0, min(V, v0 + per)


def per_shard(V: int, world: int, align: int) -> int:
    """Rows of every shard but the last non-empty one."""
    v0, v1 = shard_rows(V, world, 0, align)
    return v1 - v0


def tp_linear_logp_fwd(hidden, W_shard, targets, V, temperature, group=None):
    """logp, entropy, lse [T] of the full vocabulary from this rank's shard of
    W (rows shard_rows(V, world, rank, shard_alignment(V))), on every rank of
    `group`."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    split = binding.fwd_split_width()
    align = shard_alignment(V, split)
    v0, v1 = shard_rows(V, world, rank, align)
    if W_shard.shape[0] != v1 - v0:
        raise ValueError("W_shard must hold rows [%d, %d) of W" % (v0, v1))
    T = hidden.shape[0]
    Gs = _cdiv(per_shard(V, world, align), split)
    dev = hidden.device
    part = [torch.zeros(T, Gs, dtype=torch.float32, device=dev) for _ in range(3)]
    ytgt = torch.zeros(T, dtype=torch.float32, device=dev)
    if v1 > v0:
        binding.rlk_linear_logp_fwd_shard(hidden, W_shard, targets, V, v0, temperature, part,
                                          ytgt)
    # shards past the last vocab row hold nothing; the combine skips them
    nshards = _cdiv(_cdiv(V, split), Gs)
    gathered = []
    for p in part:
        g = torch.empty(world * T, Gs, dtype=torch.float32, device=dev)
        dist.all_gather_into_tensor(g, p, group=group)
        gathered.append(g.view(world, T, Gs)[:nshards])
    # exactly one rank owns each row's target; the others add +0
    dist.all_reduce(ytgt, group=group)
    return binding.rlk_linear_logp_combine(gathered, nshards, Gs, ytgt, targets, V)


def tp_linear_logp_bwd(hidden, W_shard, targets, V, temperature, lse, entropy, dlogp, dentropy,
                       group=None):
    """dHidden [T, H] bf16 (the same on every rank) and this rank's dW rows
    [V_shard, H] fp32, from the full-vocabulary lse and entropy of
    tp_linear_logp_fwd."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    chunk = binding.bwd_chunk_width(V)
    align = shard_alignment(V, binding.fwd_split_width(), chunk)
    v0, v1 = shard_rows(V, world, rank, align)
    if W_shard.shape[0] != v1 - v0:
        raise ValueError("W_shard must hold rows [%d, %d) of W" % (v0, v1))
    T, H = hidden.shape
    dev = hidden.device
    R = max(1, _cdiv(T, world))                     # rows of each rank's dHidden slice
    cps = _cdiv(per_shard(V, world, align), chunk)  # chunk slots per shard
    parts = torch.zeros(world, cps, R, H, dtype=torch.float32, device=dev)
    if v1 > v0:
        dW_shard, _ = binding.rlk_linear_logp_bwd_shard(hidden, W_shard, targets, V, v0,
                                                        temperature, lse, entropy, dlogp,
                                                        dentropy, parts, R)
    else:
        dW_shard = torch.zeros(0, H, dtype=torch.float32, device=dev)
    # slice q of every rank's products goes to rank q: recv[src][k] = chunk src*cps + k
    recv = torch.empty_like(parts)
    dist.all_to_all_single(recv, parts, group=group)
    # shards before the last non-empty one are full, so the first ceil(V /
    # chunk) slots in (src, k) order are the chunks in global order
    mine = torch.empty(R, H, dtype=torch.bfloat16, device=dev)
    binding.rlk_dhidden_combine(recv, _cdiv(V, chunk), mine)
    full = torch.empty(world * R, H, dtype=torch.bfloat16, device=dev)
    dist.all_gather_into_tensor(full, mine, group=group)
    return full[:T], dW_shard


class TPLinearLogp(torch.autograd.Function):
    """autograd wrapper of the vocab-parallel path:
    (logp, entropy) = TPLinearLogp.apply(hidden, W_shard, targets, V, temperature, group).
    Every rank passes the same hidden and targets and its own shard of W
    (rows shard_rows(V, world, rank, shard_alignment(V))); every rank gets the
    full-vocabulary logp and entropy, the same dHidden, and the gradient of its
    own W rows (fp32, cast to W_shard's dtype for autograd)."""

    @staticmethod
    def forward(ctx, hidden, W_shard, targets, V, temperature, group=None):
        logp, entropy, lse = tp_linear_logp_fwd(hidden, W_shard, targets, V, temperature, group)
        ctx.save_for_backward(hidden, W_shard, targets, lse, entropy)
        ctx.V, ctx.temperature, ctx.group = V, temperature, group
        return logp, entropy

    @staticmethod
    def backward(ctx, dlogp, dentropy):
        hidden, W_shard, targets, lse, entropy = ctx.saved_tensors
        dl = (dlogp if dlogp is not None else torch.zeros_like(lse)).float().contiguous()
        de = (dentropy if dentropy is not None else torch.zeros_like(lse)).float().contiguous()
        dH, dW = tp_linear_logp_bwd(hidden, W_shard, targets, ctx.V, ctx.temperature, lse,
                                    entropy, dl, de, ctx.group)
        return dH, dW.to(W_shard.dtype), None, None, None, None
