"""Short batches (rollout / decode shapes, T <= 256) run the forward with the
operands swapped (decode_fwd_kernel): 128 vocab rows per CTA, N = T rounded
up to 32, in the single-CTA MMA form up to N = 32 and the CTA-pair form
(M = 256, each CTA holding half of the N hidden rows) from N = 64.  Its logp, entropy and lse must be the pair kernel's bit for
bit, so that scoring reproduces the sampling logprob (the pages: "scoring
reproduces sampling logprob", h3-runtime-integration-b200 report, transition
gate; train/rollout logprob bitwise_equal, h100-cp-gradient.json); and they
must pass the oracle parity check on their own."""
import numpy as np
import pytest
import torch

import oracle
from invariant_lm_head_gemm_b200 import binding
from invariant_lm_head_gemm_b200 import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

SHORT_T = [1, 2, 3, 4, 15, 16, 17, 31, 32, 33, 63, 64, 65, 96, 100, 127, 128, 129, 160, 161,
           200, 224, 225, 240, 255, 256]


def _bits(a):
    return a.view(torch.int32)


@pytest.mark.parametrize("H,V,tau", [(1024, 151936, 0.7), (256, 20000, 1.0), (64, 1000, 1.3)])
def test_short_batches_equal_rows_of_a_long_batch(H, V, tau):
    base_T = 300                                   # > 256: the pair kernel
    case = gu.random_case(base_T, H, V, tau, seed=H + V)
    hid, W = gu.dev_bf16(case.hidden), gu.dev_bf16(case.W)
    tg = gu.dev(case.targets, torch.int64)
    ref = binding.rlk_linear_logp_fwd(hid, W, tg, tau)
    rng = np.random.default_rng(V)
    compared = 0
    for T in SHORT_T:
        rows = torch.from_numpy(rng.choice(base_T, size=T, replace=False)).cuda()
        rows[0] = 0                                # target = vocab entry 0
        if T > 1:
            rows[-1] = base_T - 1                  # target = last vocab entry
        got = binding.rlk_linear_logp_fwd(hid[rows].contiguous(), W, tg[rows].contiguous(), tau)
        torch.cuda.synchronize()
        for a, b, name in zip(got, ref, ("logp", "entropy", "lse")):
            assert torch.equal(_bits(a), _bits(b[rows])), (T, name)
            compared += T
    print("short-batch rows compared bitwise:", compared)


EDGE = [
    (1, 64, 1, 1.0),       # one-entry vocabulary
    (1, 64, 300, 1.0),     # a single row, V inside one W tile
    (5, 128, 513, 0.7),    # V one past a split
    (33, 192, 2000, 1.0),  # N = 64 with 31 padding rows
    (128, 64, 5000, 0.9),  # N = 128
    (32, 256, 3000, 1.0),  # the widest single-CTA form
    (33, 256, 3000, 1.0),  # the narrowest pair form: the odd CTA holds one valid row
    (200, 192, 2500, 0.8), # N = 224, ragged V
    (224, 64, 5000, 0.9),  # N = 224
    (256, 64, 5000, 0.9),  # the largest short batch, N = 256
    (129, 4096, 1537, 1.0),  # long K, N = 160
    (3, 4096, 1537, 1.0),  # long K, last split one tile and a column
]


@pytest.mark.parametrize("T,H,V,tau", EDGE)
def test_short_batch_parity_with_oracle(T, H, V, tau):
    case = gu.random_case(T, H, V, tau, seed=T * 7 + V)
    lp, en, ls = oracle.forward(case.hidden, case.W, case.targets, tau)
    out = gu.run(case.hidden, gu.dev_bf16(case.W), case.targets, tau)
    assert out["err"] == 0
    gu.assert_close_vec(out["logp"].cpu(), lp, "logp")
    gu.assert_close_vec(out["entropy"].cpu(), en, "entropy")
    gu.assert_close_vec(out["lse"].cpu(), ls, "lse")


def test_short_batch_repeats_and_out_of_range_target():
    case = gu.random_case(8, 256, 3000, 1.0, seed=99)
    hid, W = gu.dev_bf16(case.hidden), gu.dev_bf16(case.W)
    tg = gu.dev(case.targets, torch.int64)
    first = binding.rlk_linear_logp_fwd(hid, W, tg, 1.0)
    for _ in range(5):
        again = binding.rlk_linear_logp_fwd(hid, W, tg, 1.0)
        for a, b in zip(again, first):
            assert torch.equal(_bits(a), _bits(b))
    bad = tg.clone()
    bad[3] = 3000
    ws = binding.make_workspace(8, 256, 3000, False)
    lp, en, ls = binding.rlk_linear_logp_fwd(hid, W, bad, 1.0, ws)
    torch.cuda.synchronize()
    assert binding.rlk_read_device_error(ws) & 1
    assert torch.isnan(lp[3]) and not torch.isnan(torch.cat([lp[:3], lp[4:]])).any()
    assert torch.equal(_bits(en), _bits(first[1])) and torch.equal(_bits(ls), _bits(first[2]))
