"""Vocab-parallel forward and backward on one GPU: the shards of W are run one
after another (as the ranks of a TP group would run them), their results
exchanged by indexing exactly as the all-gathers / all-to-all of the TP glue
deliver them, and merged; logp, entropy, lse, dHidden and dW must equal the
single-GPU path bit for bit for every TP degree (the pages' TP2/CP4 vs TP4/CP2
runs agree bitwise: h100-cp-gradient.json, all_parameter_hash_comparisons,
gradient_norm_comparisons, tokens_equal), and the merged results of every
degree must also match the fp64 oracle within the parity tolerances: logp,
entropy and lse of every row, dHidden by relative Frobenius error, dW on
sampled vocab rows (the pages' layouts also train correctly, not only
identically)."""
import functools

import numpy as np
import pytest
import torch

import oracle
from invariant_lm_head_gemm_b200 import binding, tp
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

WORLDS = (1, 2, 3, 4, 8)
SHAPES = [(300, 256, 40000), (64, 1024, 151936), (5, 128, 1537)]


def _bits(a):
    return a.view(torch.int32) if a.dtype == torch.float32 else a.view(torch.int16)


def _case(T, H, V, tau):
    case = gu.random_case(T, H, V, tau, seed=T + V)
    return (gu.dev_bf16(case.hidden), gu.dev_bf16(case.W), gu.dev(case.targets, torch.int64),
            gu.dev(case.dlogp, torch.float32), gu.dev(case.dentropy, torch.float32))


@functools.lru_cache(maxsize=None)
def _oracle(T, H, V, tau):
    """fp64 oracle results of _case(T, H, V, tau): logp, entropy, lse, dHidden,
    and dW on sampled vocab rows (the rows' targets, both ends and a random
    set, so that every shard of every degree holds some of them)."""
    case = gu.random_case(T, H, V, tau, seed=T + V)
    z = oracle.logits(case.hidden, case.W, tau)
    lp, en, ls = oracle.softmax_stats(z, case.targets)
    dx = oracle.dlogits(z, case.targets, tau, case.dlogp, case.dentropy)
    dH = oracle.dhidden(dx, case.W)
    rng = np.random.default_rng(T + H)
    vs = np.unique(np.concatenate([case.targets, rng.choice(V, min(V, 512), replace=False),
                                   [0, V - 1]]))
    dW = oracle.dw(dx[:, vs], case.hidden)
    return dict(logp=lp, entropy=en, lse=ls, dH=dH, vs=vs, dW=dW)


def _check_fwd_against_oracle(got, ref, what):
    for a, name in zip(got, ("logp", "entropy", "lse")):
        gu.assert_close_vec(a.cpu().numpy(), ref[name], "%s %s" % (what, name))


def _check_bwd_against_oracle(dH, dW, ref, what):
    e_h = gu.rel_frob(gu.bf16_to_f64(dH), ref["dH"])
    vs = torch.from_numpy(ref["vs"]).cuda()
    e_w = gu.rel_frob(dW[vs].double().cpu().numpy(), ref["dW"])
    assert e_h <= gu.FROB_TOL and e_w <= gu.FROB_TOL, (what, e_h, e_w)


def _fwd_shards(hid, W, tg, V, tau, world, align):
    T = hid.shape[0]
    split = binding.fwd_split_width()
    Gs = -(-tp.per_shard(V, world, align) // split)
    parts = [torch.zeros(world, T, Gs, device="cuda") for _ in range(3)]
    ytgt = torch.full((T,), float("nan"), device="cuda")
    for r in range(world):
        v0, v1 = tp.shard_rows(V, world, r, align)
        if v1 > v0:
            binding.rlk_linear_logp_fwd_shard(hid, W[v0:v1].contiguous(), tg, V, v0, tau,
                                              [p[r] for p in parts], ytgt)
    nshards = -(-(-(-V // split)) // Gs)
    return binding.rlk_linear_logp_combine([p[:nshards].contiguous() for p in parts], nshards, Gs,
                                           ytgt, tg, V)


@pytest.mark.parametrize("T,H,V", SHAPES)
def test_tp_forward_any_degree_is_single_gpu_bitwise(T, H, V):
    hid, W, tg, _, _ = _case(T, H, V, 0.9)
    ref = binding.rlk_linear_logp_fwd(hid, W, tg, 0.9)
    oref = _oracle(T, H, V, 0.9)
    assert binding.fwd_split_width() == 512
    for world in WORLDS:
        # the forward alone needs only whole 512-row splits per shard
        for align in (512, tp.shard_alignment(V)):
            got = _fwd_shards(hid, W, tg, V, 0.9, world, align)
            torch.cuda.synchronize()
            for a, b, name in zip(got, ref, ("logp", "entropy", "lse")):
                assert torch.equal(_bits(a), _bits(b)), (world, align, name)
            _check_fwd_against_oracle(got, oref, "TP=%d align=%d" % (world, align))


@pytest.mark.parametrize("T,H,V", SHAPES)
def test_tp_backward_any_degree_is_single_gpu_bitwise(T, H, V):
    tau = 0.9
    hid, W, tg, dl, de = _case(T, H, V, tau)
    lp, en, ls = binding.rlk_linear_logp_fwd(hid, W, tg, tau)
    dH_ref, dW_ref = binding.rlk_linear_logp_bwd(hid, W, tg, tau, ls, en, dl, de)
    oref = _oracle(T, H, V, tau)
    chunk = binding.bwd_chunk_width(V)
    assert chunk == min(8192, -(-V // 256) * 256)
    align = tp.shard_alignment(V)
    nchunks = -(-V // chunk)
    for world in WORLDS:
        R = -(-T // world)
        cps = -(-tp.per_shard(V, world, align) // chunk)
        sent = []
        dW = torch.full_like(dW_ref, float("nan"))
        for r in range(world):
            parts = torch.zeros(world, cps, R, H, device="cuda")
            v0, v1 = tp.shard_rows(V, world, r, align)
            if v1 > v0:
                binding.rlk_linear_logp_bwd_shard(hid, W[v0:v1].contiguous(), tg, V, v0, tau, ls,
                                                  en, dl, de, parts, R, dW_shard=dW[v0:v1])
            sent.append(parts)
        slices = []
        for q in range(world):   # what the all-to-all hands rank q
            recv = torch.stack([sent[r][q] for r in range(world)]).contiguous()
            out = torch.empty(R, H, dtype=torch.bfloat16, device="cuda")
            slices.append(binding.rlk_dhidden_combine(recv, nchunks, out))
        dH = torch.cat(slices)[:T]
        torch.cuda.synchronize()
        assert torch.equal(_bits(dH), _bits(dH_ref)), world
        assert torch.equal(_bits(dW), _bits(dW_ref)), world
        _check_bwd_against_oracle(dH, dW, oref, "TP=%d" % world)


def test_plain_part_layout_and_combine():
    """part_rows = T: products laid out [chunk][T][H]; their fixed-order sum
    is dHidden, and each product is the chunk's own dX_c . W_c."""
    T, H, V, tau = 130, 128, 20000, 1.0
    hid, W, tg, dl, de = _case(T, H, V, tau)
    lp, en, ls = binding.rlk_linear_logp_fwd(hid, W, tg, tau)
    dH_ref, dW_ref = binding.rlk_linear_logp_bwd(hid, W, tg, tau, ls, en, dl, de)
    nchunks = -(-V // binding.bwd_chunk_width(V))
    parts = torch.zeros(1, nchunks, T, H, device="cuda")
    dW, _ = binding.rlk_linear_logp_bwd_shard(hid, W, tg, V, 0, tau, ls, en, dl, de, parts, T)
    dH = binding.rlk_dhidden_combine(parts, nchunks, torch.empty(T, H, dtype=torch.bfloat16,
                                                                   device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(_bits(dH), _bits(dH_ref)) and torch.equal(_bits(dW), _bits(dW_ref))
    # the products add up (in fp64) to the fp32 dHidden within rounding
    total = parts[0].double().sum(0)
    assert torch.allclose(total, dH_ref.double(), rtol=1e-2, atol=1e-3 * total.abs().max().item())


def test_shard_grid_is_enforced():
    T, H, V = 4, 64, 20000
    hid, W, tg, dl, de = _case(T, H, V, 1.0)
    parts = [torch.zeros(4, 40, device="cuda") for _ in range(3)]
    ytgt = torch.zeros(4, device="cuda")
    with pytest.raises(binding.RlkError) as e:
        binding.rlk_linear_logp_fwd_shard(hid, W[100:1000].contiguous(), tg, V, 100, 1.0, parts,
                                          ytgt)
    assert e.value.status == 2
    lse = torch.zeros(T, device="cuda")
    dp = torch.zeros(1, 3, T, H, device="cuda")
    with pytest.raises(binding.RlkError) as e:   # off the 8192-row chunk grid
        binding.rlk_linear_logp_bwd_shard(hid, W[512:9000].contiguous(), tg, V, 512, 1.0, lse,
                                          lse, lse, lse, dp, T)
    assert e.value.status == 2


def test_tp_glue_on_a_one_rank_nccl_group_matches_single_gpu():
    """The tp.py glue with its real kernels and NCCL collectives, on a group of
    one rank (the only size one GPU can hold): logp, entropy, dHidden and dW
    through TPLinearLogp equal LinearLogp's bit for bit."""
    import os
    import socket

    import torch.distributed as dist

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        T, H, V, tau = 300, 256, 20000, 0.9
        hid, W, tg, dl, de = _case(T, H, V, tau)
        h1 = hid.clone().requires_grad_(True)
        w1 = W.clone().requires_grad_(True)
        lp1, en1 = tp.TPLinearLogp.apply(h1, w1, tg, V, tau)
        (lp1 * dl + en1 * de).sum().backward()
        h2 = hid.clone().requires_grad_(True)
        w2 = W.clone().requires_grad_(True)
        lp2, en2 = binding.LinearLogp.apply(h2, w2, tg, tau)
        (lp2 * dl + en2 * de).sum().backward()
        torch.cuda.synchronize()
        assert torch.equal(_bits(lp1.detach()), _bits(lp2.detach()))
        assert torch.equal(_bits(en1.detach()), _bits(en2.detach()))
        assert torch.equal(_bits(h1.grad), _bits(h2.grad))
        assert torch.equal(_bits(w1.grad), _bits(w2.grad))
    finally:
        dist.destroy_process_group()
