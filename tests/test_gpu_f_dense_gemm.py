"""Batch-invariant deterministic dense GEMM (the FFN / LoRA-gate core) through
rlk_gemm_bf16_f32, on the shapes of the pages' LoRA gate
(h3-runtime-integration-b200 report, lora_gate[].shape: N512 K384 T70,
N2048 K1024 T257, N5120 K5120 T33) and its checks: repeatable,
forward_rows_independent, and the error against fp64.  The gate reports
~1.66e-3 relative error for bf16 outputs; this GEMM returns fp32, so its own
error is far smaller, and rounding its output to bf16 lands near the gate's
figure."""
import json
import os

import pytest
import torch

from invariant_lm_head_gemm_b200 import binding

pytestmark = pytest.mark.gpu

with open(os.path.join(os.path.dirname(__file__), "golden", "pages_claims.json")) as _f:
    LORA_FWD_ERR = json.load(_f)["lora_gate_forward_rel_err_vs_fp64"]["values"]

SHAPES = [(512, 384, 70), (2048, 1024, 257), (5120, 5120, 33)]   # (N, K, T)


def _rel(a, b):
    return float((a.double() - b).norm() / b.norm())


@pytest.mark.parametrize("N,K,T", SHAPES, ids=lambda *a: None)
def test_gate_shapes(N, K, T):
    g = torch.Generator().manual_seed(N + K + T)
    x = torch.randn(T, K, generator=g).to(torch.bfloat16)
    W = (torch.randn(N, K, generator=g) / K ** 0.5).to(torch.bfloat16)
    xd, Wd = x.cuda(), W.cuda()
    y, ws = binding.rlk_gemm_bf16_f32(xd, Wd)
    y2, _ = binding.rlk_gemm_bf16_f32(xd, Wd)
    torch.cuda.synchronize()
    assert binding.rlk_read_device_error(ws) == 0
    # repeatable
    assert torch.equal(y.view(torch.int32), y2.view(torch.int32))
    ref = x.double() @ W.double().t()
    err = _rel(y.cpu(), ref)
    assert err < 1e-5, err
    # rounded to bf16 the error is that of a bf16-output GEMM, the gate's figure
    err_bf16 = _rel(y.cpu().to(torch.bfloat16).float(), ref)
    assert err_bf16 < 2 * max(LORA_FWD_ERR), err_bf16
    # rows independent of the rest of the batch: any subset of rows gives the
    # same bits for those rows
    for rows in ([0], [T - 1], list(range(0, T, 3)), list(range(T - 1, -1, -2))):
        idx = torch.tensor(rows)
        sub, _ = binding.rlk_gemm_bf16_f32(xd[idx].contiguous(), Wd)
        torch.cuda.synchronize()
        assert torch.equal(sub.view(torch.int32), y[idx.cuda()].view(torch.int32)), rows
    print((N, K, T), "rel err fp32 %.2e, as bf16 %.2e (gate: %.2e)" % (err, err_bf16, LORA_FWD_ERR[0]))
