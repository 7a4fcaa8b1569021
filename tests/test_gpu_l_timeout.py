"""The fail-closed path of a wait that never ends: every wait inside the
kernels is bounded, and when one gives up the kernel records
RLK_DEVERR_TIMEOUT in the workspace, lets its in-flight copies and MMAs finish,
frees its tensor memory and returns, so the context stays usable and the next
call behaves as on a fresh workspace (the pages' runs require an error status,
not a hang: VIME Qwen3-8B TP4/CP2 page, "Required gates";
h3-runtime-integration-b200 report, fail_on_fallback).  The stall is a
dependency counter target that nothing reaches (a test hook of the library),
with a 100 ms bound on every wait; nothing faults, traps or hangs."""
import time

import pytest
import torch

from invariant_lm_head_gemm_b200 import binding
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

LIMIT_NS = 100_000_000  # 100 ms


def _bits(t):
    return t.view(torch.int32) if t.dtype == torch.float32 else t.view(torch.int16)


def test_stalled_backward_reports_timeout_and_the_next_call_is_unaffected():
    tau = 0.9
    case = gu.random_case(300, 256, 40000, tau, seed=909)
    hid, W = gu.dev_bf16(case.hidden), gu.dev_bf16(case.W)
    tg = gu.dev(case.targets, torch.int64)
    dl, de = gu.dev(case.dlogp, torch.float32), gu.dev(case.dentropy, torch.float32)
    T, H, V = case.T, case.H, case.V
    ws = binding.make_workspace(T, H, V, True)
    lp, en, ls = binding.rlk_linear_logp_fwd(hid, W, tg, tau, ws)
    dH_ref, dW_ref = (t.clone() for t in binding.rlk_linear_logp_bwd(hid, W, tg, tau, ls, en,
                                                                     dl, de, ws))
    torch.cuda.synchronize()
    assert binding.rlk_read_device_error(ws) == 0

    out = (torch.empty(T, H, dtype=torch.bfloat16, device="cuda"),
           torch.empty(V, H, device="cuda"))
    # the short bound alone changes nothing
    binding.rlk_test_linear_logp_bwd_stall(hid, W, tg, tau, ls, en, dl, de, ws, out, LIMIT_NS, 0)
    torch.cuda.synchronize()
    assert binding.rlk_read_device_error(ws) == 0
    assert torch.equal(_bits(out[0]), _bits(dH_ref)) and torch.equal(_bits(out[1]), _bits(dW_ref))

    # a dependency nothing meets: the call returns, the error word says timeout,
    # and every vocab-chunk completion word is published anyway, so a stream
    # waiting on them (an overlapped dW exchange) is released
    nchunks = -(-V // binding.bwd_chunk_width(V))
    words = torch.zeros(nchunks, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    binding.rlk_test_linear_logp_bwd_stall(hid, W, tg, tau, ls, en, dl, de, ws, out, LIMIT_NS, 1,
                                           chunk_done=words, seq=5)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    flags = binding.rlk_read_device_error(ws)
    assert flags & binding.RLK_DEVERR_TIMEOUT, flags
    assert elapsed < 60.0, elapsed
    assert (words == 5).all()
    side = torch.cuda.Stream()
    for c in range(nchunks):
        binding.rlk_stream_wait_chunk(words[c:c + 1], 5, side)
    side.synchronize()

    # the next calls on the same workspace and stream are bit for bit those of
    # a fresh run
    dH2, dW2 = binding.rlk_linear_logp_bwd(hid, W, tg, tau, ls, en, dl, de, ws)
    lp2, en2, ls2 = binding.rlk_linear_logp_fwd(hid, W, tg, tau, ws)
    torch.cuda.synchronize()
    assert binding.rlk_read_device_error(ws) == 0
    assert torch.equal(_bits(dH2), _bits(dH_ref)) and torch.equal(_bits(dW2), _bits(dW_ref))
    for a, b in ((lp2, lp), (en2, en), (ls2, ls)):
        assert torch.equal(_bits(a), _bits(b))



@pytest.mark.parametrize("T", [16, 128, 200, 256])
def test_stalled_short_batch_forward_reports_timeout_and_the_next_call_is_unaffected(T):
    """The short-batch forward (single-CTA MMA form at T = 16, CTA-pair form at
    T = 128, 200 and 256) with the first CTA of every cluster waiting for an
    accumulator that never reports full: its epilogue, the chain of the other
    three CTAs and the MMA issuer run out their 100 ms waits, the call returns,
    the error word says timeout, and the next calls on the same workspace give
    the results of a fresh one bit for bit."""
    tau = 1.0
    case = gu.random_case(T, 256, 20000, tau, seed=T + 77)
    hid, W = gu.dev_bf16(case.hidden), gu.dev_bf16(case.W)
    tg = gu.dev(case.targets, torch.int64)
    ws = binding.make_workspace(T, 256, 20000, False)
    ref = [t.clone() for t in binding.rlk_linear_logp_fwd(hid, W, tg, tau, ws)]
    torch.cuda.synchronize()
    assert binding.rlk_read_device_error(ws) == 0
    out = tuple(torch.empty(T, device="cuda") for _ in range(3))
    # the short bound alone changes nothing
    binding.rlk_test_linear_logp_fwd_stall(hid, W, tg, tau, ws, out, LIMIT_NS, 0)
    torch.cuda.synchronize()
    assert binding.rlk_read_device_error(ws) == 0
    for a, b in zip(out, ref):
        assert torch.equal(_bits(a), _bits(b))
    t0 = time.perf_counter()
    binding.rlk_test_linear_logp_fwd_stall(hid, W, tg, tau, ws, out, LIMIT_NS, 1)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    flags = binding.rlk_read_device_error(ws)
    assert flags & binding.RLK_DEVERR_TIMEOUT, flags
    assert elapsed < 5.0, elapsed   # a few 100 ms bounds in a chain, not the 2 s default
    for _ in range(2):
        again = binding.rlk_linear_logp_fwd(hid, W, tg, tau, ws)
        torch.cuda.synchronize()
        assert binding.rlk_read_device_error(ws) == 0
        for a, b in zip(again, ref):
            assert torch.equal(_bits(a), _bits(b))
