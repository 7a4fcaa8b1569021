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
