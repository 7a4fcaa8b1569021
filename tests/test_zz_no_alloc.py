"""The forward entry point that takes no workspace and allocates nothing, for
callers that cannot allocate device memory (their host framework owns every
device byte, or they cannot size a workspace ahead of time).  Its scratch is a
fixed device array inside the library, shared by every call.

Checked through the C ABI against the workspace entry point, on two calls in
a row with different shapes (the second call must not see the first call's
leftovers), plus the size limit.  Collected last on purpose, and written to
pass alone in a fresh process as well as after the other tests."""
import ctypes

import numpy as np
import pytest
import torch

from invariant_lm_head_gemm_b200 import binding
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def _compare(case):
    W_dev = gu.dev_bf16(case.W)
    hid = gu.dev_bf16(case.hidden)
    tg = gu.dev(case.targets, torch.int64)
    ref = binding.rlk_linear_logp_fwd(hid, W_dev, tg, case.temperature)
    got = binding.rlk_linear_logp_fwd_noalloc(hid, W_dev, tg, case.temperature)
    torch.cuda.synchronize()
    for name, g, r in zip(("logp", "entropy", "lse"), got, ref):
        gu.assert_close_vec(g.cpu().numpy(), r.cpu().numpy(), name)
    return got


def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row():
    first = gu.random_case(300, 256, 20000, 0.9, seed=301)
    second = gu.random_case(37, 128, 1000, 1.0, seed=302)
    a = _compare(first)
    b = _compare(second)
    assert a[0].shape[0] == 300 and b[0].shape[0] == 37
    assert all(torch.isfinite(x).all() for x in a + b)


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
