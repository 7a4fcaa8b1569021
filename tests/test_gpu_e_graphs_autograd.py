"""CUDA-graph capture and the autograd wrapper.

The pages validate vLLM CUDA-graph capture of the decode path with capture
sizes 1..4 (h100-cp-gradient.json, runs[0].validation.cudagraph:
expected_capture_sizes [1, 2, 3, 4]); the library enqueues everything on the
caller's stream and allocates nothing, so both passes must capture into a
graph and replay bit for bit like eager calls."""
import json
import os

import numpy as np
import pytest
import torch

from invariant_lm_head_gemm_b200 import binding
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

with open(os.path.join(os.path.dirname(__file__), "golden", "pages_claims.json")) as _f:
    CAPTURE_SIZES = json.load(_f)["cudagraph_expected_capture_sizes"]["sizes"]


def _same_bits(a, b):
    it = {torch.float32: torch.int32, torch.bfloat16: torch.int16}[a.dtype]
    return torch.equal(a.view(it), b.view(it))


def _tensors(case):
    hid = gu.dev_bf16(case.hidden)
    W = gu.dev_bf16(case.W)
    tg = gu.dev(case.targets, torch.int64)
    dl = gu.dev(case.dlogp, torch.float32)
    de = gu.dev(case.dentropy, torch.float32)
    return hid, W, tg, dl, de


def _outputs(T, H, V):
    return ([torch.empty(T, device="cuda") for _ in range(3)],
            (torch.empty(T, H, dtype=torch.bfloat16, device="cuda"),
             torch.empty(V, H, device="cuda")))


@pytest.mark.parametrize("T", CAPTURE_SIZES + [300])
def test_capture_and_replay_match_eager(T):
    H, V = 256, 20000
    case = gu.random_case(T, H, V, 1.0, seed=500 + T)
    hid, W, tg, dl, de = _tensors(case)
    ws = binding.make_workspace(T, H, V, True)
    (e_lp, e_en, e_ls), (e_dH, e_dW) = _outputs(T, H, V)
    binding.rlk_linear_logp_fwd(hid, W, tg, 1.0, ws, out=(e_lp, e_en, e_ls))
    binding.rlk_linear_logp_bwd(hid, W, tg, 1.0, e_ls, e_en, dl, de, ws, out=(e_dH, e_dW))
    torch.cuda.synchronize()

    (g_lp, g_en, g_ls), (g_dH, g_dW) = _outputs(T, H, V)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        binding.rlk_linear_logp_fwd(hid, W, tg, 1.0, ws, out=(g_lp, g_en, g_ls))
        binding.rlk_linear_logp_bwd(hid, W, tg, 1.0, g_ls, g_en, dl, de, ws, out=(g_dH, g_dW))
    for _ in range(2):
        for t in (g_lp, g_en, g_ls, g_dW):
            t.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        for a, b in ((g_lp, e_lp), (g_en, e_en), (g_ls, e_ls), (g_dH, e_dH), (g_dW, e_dW)):
            assert _same_bits(a, b)
    assert binding.rlk_read_device_error(ws) == 0


def test_autograd_wrapper_matches_direct_calls():
    T, H, V = 70, 256, 5000
    case = gu.random_case(T, H, V, 0.8, seed=611)
    hid, W, tg, dl, de = _tensors(case)
    h = hid.clone().requires_grad_(True)
    w = W.float().clone().to(torch.bfloat16).requires_grad_(True)
    logp, ent = binding.LinearLogp.apply(h, w, tg, 0.8)
    (logp * dl + ent * de).sum().backward()
    lp, en, ls = binding.rlk_linear_logp_fwd(hid, W, tg, 0.8)
    dH, dW = binding.rlk_linear_logp_bwd(hid, W, tg, 0.8, ls, en, dl, de)
    torch.cuda.synchronize()
    assert _same_bits(logp.detach(), lp) and _same_bits(ent.detach(), en)
    assert _same_bits(h.grad, dH)
    # the wrapper casts dW (fp32) to W's dtype for autograd
    assert torch.equal(w.grad, dW.to(torch.bfloat16))
    assert np.isfinite(h.grad.float().cpu().numpy()).all()
