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
