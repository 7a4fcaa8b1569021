"""The forward entry point that takes no workspace and allocates nothing, for
callers that cannot allocate device memory (their host framework owns every
device byte, or they cannot size a workspace ahead of time).  Its scratch is a
fixed device array inside the library, shared by every call.

Checked through the C ABI against the workspace entry point, bit for bit, on
two calls in a row with different shapes (the second call must not see the
first call's leftovers), with an out-of-range target in the second call; the
device's free memory must not move across calls once the first call has run;
and the size limit.  Collected last on purpose, and written to pass alone in a
fresh process as well as after the other tests."""
import ctypes

import pytest
import torch

from invariant_lm_head_gemm_b200 import binding
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def _inputs(case, bad_row=None):
    W_dev = gu.dev_bf16(case.W)
    hid = gu.dev_bf16(case.hidden)
    tg = gu.dev(case.targets, torch.int64)
    if bad_row is not None:
        tg[bad_row] = case.W.shape[0]  # target == V: out of range
    return hid, W_dev, tg


def _bits(t):
    return t.view(torch.int32)


def _compare(case, bad_row=None):
    hid, W_dev, tg = _inputs(case, bad_row)
    ref = binding.rlk_linear_logp_fwd(hid, W_dev, tg, case.temperature)
    got = binding.rlk_linear_logp_fwd_noalloc(hid, W_dev, tg, case.temperature)
    torch.cuda.synchronize()
    for name, g, r in zip(("logp", "entropy", "lse"), got, ref):
        assert torch.equal(_bits(g), _bits(r)), name  # same kernels: same bits
    # and the workspace entry is itself within tolerance of the oracle-checked
    # results the rest of the suite pins; here the two entries must agree
    return got


def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row():
    first = gu.random_case(300, 256, 20000, 0.9, seed=301)
    second = gu.random_case(37, 128, 1000, 1.0, seed=302)
    c0 = binding.call_count(0)
    a = _compare(first)
    b = _compare(second, bad_row=5)
    # each _compare makes one workspace call and one no-allocation call
    assert binding.call_count(0) == c0 + 4
    assert a[0].shape[0] == 300 and b[0].shape[0] == 37
    assert all(torch.isfinite(x).all() for x in a)
    logp, ent, lse = b
    assert torch.isnan(logp[5])
    keep = torch.ones(37, dtype=torch.bool, device=logp.device)
    keep[5] = False
    assert torch.isfinite(logp[keep]).all()
    assert torch.isfinite(ent).all() and torch.isfinite(lse).all()


def test_noalloc_allocates_no_device_memory():
    case = gu.random_case(129, 256, 5000, 1.0, seed=303)
    hid, W_dev, tg = _inputs(case)
    outs = tuple(torch.empty(case.hidden.shape[0], device="cuda") for _ in range(3))
    binding.rlk_linear_logp_fwd_noalloc(hid, W_dev, tg, 1.0, out=outs)  # module loaded now
    torch.cuda.synchronize()
    first = [t.clone() for t in outs]
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        binding.rlk_linear_logp_fwd_noalloc(hid, W_dev, tg, 1.0, out=outs)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    for a, b in zip(outs, first):
        assert torch.equal(_bits(a), _bits(b))


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # validation happens before anything touches the device: these pointers
    # are never dereferenced
    f = binding.lib().rlk_linear_logp_fwd_noalloc
    f.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64] * 3 + [ctypes.c_float] + \
        [ctypes.c_void_p] * 4
    f.restype = ctypes.c_int
    p = 0x10000
    assert f(p, p, p, 20000, 4096, 151936, 1.0, p, p, p, None) == 4   # WORKSPACE_TOO_SMALL
    assert f(p, p, p, 4, 100, 10, 1.0, p, p, p, None) == 2            # UNSUPPORTED_SHAPE
