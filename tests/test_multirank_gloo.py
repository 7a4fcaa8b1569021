"""The multi-GPU host logic on CPU: two gloo ranks.  Rows are independent, so
ranks share no data; what must hold is the per-rank workload (each rank its
own batch against the same W) and the aggregation (slowest rank's time,
all ranks' tokens)."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    from invariant_lm_head_gemm_b200 import workloads as wl
    ms, tokens = bench.aggregate(10.0 + rank, 100 * (rank + 1))
    w = wl.rl_step(3 + 1000 * rank, with_weight=False)
    out[rank] = (ms, tokens, int(w.T), float(w.hidden[:4, :4].astype(np.float64).sum()))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_gloo_ranks_aggregate_and_shard():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][:2] == (11.0, 300.0) and res[1][:2] == (11.0, 300.0)
    # each rank draws its own batch (different sequence lengths and rows)
    assert res[0][2:] != res[1][2:]


def test_single_process_aggregate_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate(12.5, 5980) == (12.5, 5980.0)


def _dw(rank, V, H):
    import torch
    g = torch.Generator().manual_seed(1000 + rank)
    return torch.randn(V, H, generator=g)


def _cpu_ordered_sum(parts, out):
    acc = parts[0].clone()
    for p in parts[1:]:
        acc = acc + p
    out.copy_(acc)


def _rs_worker(rank, world, port, V, H, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    from invariant_lm_head_gemm_b200 import dp
    res, r0, r1 = dp.reduce_scatter_dw(_dw(rank, V, H), sum_fn=_cpu_ordered_sum)
    out[rank] = (r0, r1, res.numpy().tobytes())
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world,V", [(2, 37), (3, 8), (2, 1)])
def test_dw_reduce_scatter_is_the_rank_ordered_sum(world, V):
    H = 8
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rs_worker, args=(world, _free_port(), V, H, out), nprocs=world, join=True)
        res = dict(out)
    full = _dw(0, V, H)
    for r in range(1, world):
        full = full + _dw(r, V, H)          # rank order
    covered = 0
    for r in range(world):
        r0, r1, raw = res[r]
        got = np.frombuffer(raw, dtype=np.float32).reshape(-1, H)[: r1 - r0]
        assert np.array_equal(got.view(np.uint32), full[r0:r1].numpy().view(np.uint32))
        covered += r1 - r0
    assert covered == V


def _tp_worker(rank, world, port, V, T, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    from invariant_lm_head_gemm_b200 import binding, tp
    # stand-ins for the CUDA entry points: record what the glue hands over
    seen = {}

    def fake_shard(hidden, W_shard, targets, V_, v0, temperature, part, ytgt, workspace=None,
                   stream=None):
        for k, p in enumerate(part):
            p.copy_(torch.full_like(p, 100 * rank + k))
        owned = (targets >= v0) & (targets < v0 + W_shard.shape[0])
        ytgt[owned] = targets[owned].float()

    def fake_combine(part, nshards, Gs, ytgt, targets, V_, out=None, workspace=None, stream=None):
        seen.update(nshards=nshards, Gs=Gs, part=[p.clone() for p in part], ytgt=ytgt.clone())
        return None

    binding.fwd_split_width = lambda: 512
    binding.bwd_chunk_width = lambda V_: 8192
    binding.rlk_linear_logp_fwd_shard = fake_shard
    binding.rlk_linear_logp_combine = fake_combine
    v0, v1 = tp.shard_rows(V, world, rank, tp.shard_alignment(V))
    targets = torch.arange(T, dtype=torch.int64) * (V // T)
    tp.tp_linear_logp_fwd(torch.zeros(T, 64), torch.zeros(v1 - v0, 64), targets, V, 1.0)
    out[rank] = (v0, v1, seen["nshards"], seen["Gs"],
                 [p[:, 0, 0].tolist() for p in seen["part"]], seen["ytgt"].tolist())
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_tp_glue_gathers_shards_in_rank_order():
    world, V, T = 3, 151936, 6
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_tp_worker, args=(world, _free_port(), V, T, out), nprocs=world, join=True)
        res = dict(out)
    bounds = [res[r][:2] for r in range(world)]
    assert bounds[0][0] == 0 and bounds[-1][1] == V
    assert all(b[0] % 8192 == 0 for b in bounds)
    assert all(bounds[r][1] == bounds[r + 1][0] for r in range(world - 1))
    for r in range(world):
        _, _, nshards, Gs, parts, ytgt = res[r]
        assert nshards == world and (nshards - 1) * Gs < -(-V // 512) <= nshards * Gs
        for k in range(3):                       # shard r's triples at position r
            assert parts[k] == [100 * q + k for q in range(world)]
        assert ytgt == [float(t * (V // T)) for t in range(T)]   # every row owned once


def _tp_bwd_worker(rank, world, port, V, T, H, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    from invariant_lm_head_gemm_b200 import binding, tp
    seen = {}

    def fake_bwd_shard(hidden, W_shard, targets, V_, v0, tau, lse, ent, dl, de, parts, R,
                       dW_shard=None, workspace=None, stream=None):
        # value = 1000 * rank + 100 * slice + 10 * local chunk + local row
        S, cps, R_, H_ = parts.shape
        nloc = -(-W_shard.shape[0] // 8192)
        for s in range(S):
            for k in range(nloc):
                for r in range(R_):
                    parts[s, k, r] = 1000 * rank + 100 * s + 10 * k + r
        return torch.full((W_shard.shape[0], H_), float(rank)), None

    def fake_combine(parts, nparts, out, stream=None):
        seen.update(nparts=nparts, recv=parts.clone())
        out.copy_(torch.full_like(out, rank))
        return out

    binding.fwd_split_width = lambda: 512
    binding.bwd_chunk_width = lambda V_: 8192
    binding.rlk_linear_logp_bwd_shard = fake_bwd_shard
    binding.rlk_dhidden_combine = fake_combine
    v0, v1 = tp.shard_rows(V, world, rank, tp.shard_alignment(V))
    z = torch.zeros(T)
    dH, dW = tp.tp_linear_logp_bwd(torch.zeros(T, H, dtype=torch.bfloat16),
                                   torch.zeros(v1 - v0, H), torch.zeros(T, dtype=torch.int64), V,
                                   1.0, z, z, z, z)
    out[rank] = (v0, v1, seen["nparts"], seen["recv"][:, :, :, 0].tolist(),
                 dH[:, 0].float().tolist(), list(dW.shape))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world,V,T", [(3, 40000, 7), (2, 151936, 4), (4, 20000, 3)])
def test_tp_backward_glue_routes_chunk_products(world, V, T):
    H = 4
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_tp_bwd_worker, args=(world, _free_port(), V, T, H, out), nprocs=world,
                 join=True)
        res = dict(out)
    R = -(-T // world)
    nchunks = -(-V // 8192)
    owners = []          # (rank, local chunk) of every global chunk, in order
    for r in range(world):
        v0, v1 = res[r][:2]
        assert v1 == v0 or (v0 % 8192 == 0 and (v1 == V or (v1 - v0) % 8192 == 0))
        owners += [(r, k) for k in range(-(-(v1 - v0) // 8192))]
        assert res[r][5] == [v1 - v0, H]
    assert len(owners) == nchunks
    for q in range(world):
        _, _, nparts, recv, dH, _ = res[q]
        assert nparts == nchunks
        cps = len(recv[0])
        flat = [recv[src][k] for src in range(world) for k in range(cps)]
        # the first nchunks blocks are the chunks in global order, each holding
        # row slice q of its owner's product
        for g, (src, k) in enumerate(owners):
            assert flat[g] == [1000 * src + 100 * q + 10 * k + r for r in range(R)], (q, g)
        # dHidden rows come back in rank order, the padding rows dropped
        assert dH == [float(t // R) for t in range(T)]


def _tp_autograd_worker(rank, world, port, V, T, H, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    from invariant_lm_head_gemm_b200 import tp
    calls = []

    def fake_fwd(hidden, W_shard, targets, V_, tau, group=None):
        calls.append(("fwd", W_shard.shape[0]))
        T_ = hidden.shape[0]
        return (torch.full((T_,), -1.0 - rank), torch.full((T_,), 2.0), torch.full((T_,), 3.0))

    def fake_bwd(hidden, W_shard, targets, V_, tau, lse, entropy, dl, de, group=None):
        calls.append(("bwd", float(lse[0]), float(entropy[0]), float(dl[0]), float(de[0])))
        return torch.full_like(hidden, 5.0), torch.full((W_shard.shape[0], hidden.shape[1]), 7.0)

    tp.tp_linear_logp_fwd = fake_fwd
    tp.tp_linear_logp_bwd = fake_bwd
    h = torch.zeros(T, H, requires_grad=True)
    w = torch.zeros(11 + rank, H, requires_grad=True)
    logp, ent = tp.TPLinearLogp.apply(h, w, torch.zeros(T, dtype=torch.int64), V, 1.0)
    (logp * 0.5 + ent * 0.25).sum().backward()
    out[rank] = (calls, float(h.grad[0, 0]), list(w.grad.shape), float(w.grad[0, 0]),
                 float(logp[0]))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_tp_autograd_wrapper_plumbing():
    world, V, T, H = 2, 20000, 3, 4
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_tp_autograd_worker, args=(world, _free_port(), V, T, H, out), nprocs=world,
                 join=True)
        res = dict(out)
    for r in range(world):
        calls, dh, wshape, dw, lp0 = res[r]
        assert calls[0] == ("fwd", 11 + r)
        # backward receives the saved lse / entropy and the upstream gradients
        assert calls[1] == ("bwd", 3.0, 2.0, 0.5, 0.25)
        assert dh == 5.0 and wshape == [11 + r, H] and dw == 7.0 and lp0 == -1.0 - r


def _rs_overlap_worker(rank, world, port, V, H, chunk, gc, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    from invariant_lm_head_gemm_b200 import dp
    waited = []
    res, pieces = dp.reduce_scatter_dw_overlapped(
        _dw(rank, V, H), chunk, chunk_done=list(range(100)), seq=7, group_chunks=gc,
        sum_fn=_cpu_ordered_sum, wait_fn=lambda word, seq, stream: waited.append((word, seq)))
    out[rank] = (pieces, res.numpy().tobytes(), waited)
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world,V,chunk,gc", [(2, 37, 8, 2), (3, 70, 16, 1), (2, 5, 8, 4),
                                              (3, 100, 8, 3)])
def test_overlapped_dw_exchange_is_the_rank_ordered_sum(world, V, chunk, gc):
    """The chunk-group exchange: every rank's pieces hold the rank-ordered sum
    of those rows bit for bit, the pieces of all ranks cover [0, V) once, and
    each group waits for every one of its chunks (in order) before it moves."""
    H = 4
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rs_overlap_worker, args=(world, _free_port(), V, H, chunk, gc, out),
                 nprocs=world, join=True)
        res = dict(out)
    full = _dw(0, V, H)
    for r in range(1, world):
        full = full + _dw(r, V, H)          # rank order
    seen = np.zeros(V, dtype=int)
    nchunks = -(-V // chunk)
    for r in range(world):
        pieces, raw, waited = res[r]
        got = np.frombuffer(raw, dtype=np.float32).reshape(-1, H)
        off = 0
        for r0, r1 in pieces:
            assert np.array_equal(got[off:off + r1 - r0].view(np.uint32),
                                  full[r0:r1].numpy().view(np.uint32))
            seen[r0:r1] += 1
            off += r1 - r0
        assert waited == [([c], 7) for c in range(nchunks)]
    assert (seen == 1).all()
