"""C-ABI checks that need no GPU: the library builds, loads and exports every
function include/rlk.h declares; argument validation returns the documented
status before any CUDA work; provenance strings."""
import ctypes

import pytest
import torch

from invariant_lm_head_gemm_b200 import binding, build

OK, INVALID, SHAPE, MISALIGNED, WS_SMALL, DEVICE, CUDA = range(7)


@pytest.fixture(scope="module")
def L():
    build.build()
    return binding.lib()


def test_exports_every_declared_function(L):
    names = binding.declared_functions()
    assert {"rlk_linear_logp_fwd", "rlk_linear_logp_bwd",
            "rlk_linear_logp_workspace_bytes"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings_and_backend_id(L):
    assert [binding.status_string(s) for s in range(7)] == [
        "RLK_OK", "RLK_ERR_INVALID_ARG", "RLK_ERR_UNSUPPORTED_SHAPE", "RLK_ERR_MISALIGNED",
        "RLK_ERR_WORKSPACE_TOO_SMALL", "RLK_ERR_UNSUPPORTED_DEVICE", "RLK_ERR_CUDA"]
    assert binding.status_string(99) == "RLK_ERR_UNKNOWN"
    assert binding.backend_id() == "rlk.linear_logp.bitwise.sm100a.v1"
    assert binding.call_count(7) == 0


def test_workspace_bytes(L):
    T, H, V = 5200, 4096, 151936
    fwd = binding.workspace_bytes(T, H, V, False)
    both = binding.workspace_bytes(T, H, V, True)
    # fwd: 256-byte header + 3 x [297 splits x T] fp32 partials + [T] target logits
    def a(x):
        return (x + 255) // 256 * 256
    assert fwd == 256 + 3 * a(297 * T * 4) + a(T * 4)
    # bwd: header + 3 x [T, 8192] bf16 dlogits chunk buffers + [T, H] fp32 dHidden
    # accumulator + the fused backward's dependency counters
    NC, MT, NH, RT = 19, (T + 255) // 256, H // 256, 8192 // 256
    counters = NC * MT + NC * RT + NC * MT * NH + NC + 1
    assert both == max(fwd, 256 + 3 * a(T * 8192 * 2) + a(T * H * 4) + a(counters * 4))
    assert binding.workspace_bytes(4, 100, 10) == 0          # H % 64 != 0
    assert binding.workspace_bytes(4, 64, 0) == 0
    assert binding.workspace_bytes(0, 64, 10) > 0
    # small V: the chunk buffer shrinks to V rounded up to 256 columns
    assert binding.workspace_bytes(8, 64, 300, True) >= 256 + 3 * 8 * 512 * 2 + 8 * 64 * 4


A16 = 0x10000        # fake, never dereferenced: validation must fail first
A256 = 0x20000


def _fwd(L, hidden=A16, W=A16, targets=A16, T=4, H=64, V=10, tau=1.0, logp=A16, ent=A16,
         lse=A16, ws=A256, wsb=1 << 30):
    return L.rlk_linear_logp_fwd(hidden, W, targets, T, H, V, tau, logp, ent, lse, ws, wsb, None)


def _bwd(L, dW=A16, dH=A16, T=4, H=64, V=10, tau=1.0, ws=A256, wsb=1 << 30, hidden=A16):
    return L.rlk_linear_logp_bwd(hidden, A16, A16, T, H, V, tau, A16, A16, A16, A16, dH, dW,
                                 ws, wsb, None)


def test_forward_argument_errors(L):
    assert _fwd(L, T=-1) == INVALID
    assert _fwd(L, H=0) == INVALID
    assert _fwd(L, V=0) == INVALID
    for tau in (0.0, -1.0, float("nan"), float("inf"), 1e-45):
        assert _fwd(L, tau=tau) == INVALID, tau
    assert _fwd(L, H=100) == SHAPE
    assert _fwd(L, H=64 * (1 << 15)) == SHAPE
    assert _fwd(L, V=1 << 31) == SHAPE
    assert _fwd(L, T=0, hidden=None, W=None, targets=None) == OK     # empty batch: no-op
    for k in ("hidden", "W", "targets", "logp", "ent", "lse", "ws"):
        assert _fwd(L, **{k: None}) == INVALID, k
    assert _fwd(L, hidden=A16 + 8) == MISALIGNED
    assert _fwd(L, W=A16 + 2) == MISALIGNED
    assert _fwd(L, ws=A256 + 16) == MISALIGNED
    assert _fwd(L, targets=A16 + 4) == MISALIGNED
    assert _fwd(L, logp=A16 + 2) == MISALIGNED
    need = binding.workspace_bytes(4, 64, 10, False)
    assert _fwd(L, wsb=need - 1) == WS_SMALL


def test_backward_argument_errors(L):
    assert _bwd(L, T=-2) == INVALID
    assert _bwd(L, tau=0.0) == INVALID
    assert _bwd(L, H=96) == SHAPE
    assert _bwd(L, dW=None) == INVALID
    assert _bwd(L, dW=A16 + 4) == MISALIGNED
    assert _bwd(L, dH=None) == INVALID
    assert _bwd(L, hidden=None) == INVALID
    assert _bwd(L, dH=A16 + 2) == MISALIGNED
    need = binding.workspace_bytes(4, 64, 10, True)
    assert _bwd(L, wsb=need - 1) == WS_SMALL


def test_gemm_argument_errors(L):
    g = L.rlk_gemm_bf16_f32
    assert g(A16, A16, 0, 8, 8, 0, 0, A16, A256, 256, None) == INVALID
    assert g(A16, A16, 12, 8, 8, 1, 0, A16, A256, 256, None) == SHAPE    # MN-major A: M % 8
    assert g(A16, A16, 8, 12, 8, 0, 0, A16, A256, 256, None) == SHAPE    # N % 8
    assert g(A16, A16, 8, 8, 12, 0, 0, A16, A256, 256, None) == SHAPE    # K % 8
    assert g(None, A16, 8, 8, 8, 0, 0, A16, A256, 256, None) == INVALID
    assert g(A16 + 2, A16, 8, 8, 8, 0, 0, A16, A256, 256, None) == MISALIGNED
    assert g(A16, A16, 8, 8, 8, 0, 0, A16, A256, 255, None) == WS_SMALL
    v = ctypes.c_uint32(0)
    assert L.rlk_read_device_error(None, ctypes.byref(v), None) == INVALID


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU refusal")
def test_valid_call_without_a_gpu_is_refused(L):
    # every argument is valid, so the only thing left to fail is the device:
    # the library must refuse (fail closed), not fall back to anything
    assert _fwd(L) == DEVICE
    assert _bwd(L) == DEVICE
    assert _bwd(L, T=0) == DEVICE
    assert L.rlk_gemm_bf16_f32(A16, A16, 8, 8, 8, 0, 0, A16, A256, 256, None) == DEVICE
    assert _shard(L) == DEVICE and _combine(L) == DEVICE
    assert _bshard(L) == DEVICE and L.rlk_dhidden_combine(A16, 2, 8, A16, None) == DEVICE
    binding._tr()
    assert L.rlk_transition_sample(A16, A16, A16, A16, A16, A16, 2, 8, None, A16, A16, A256,
                                   1 << 20, None) == DEVICE
    assert binding.call_count(0) == 0 and binding.call_count(1) == 0


def _shard(L, v0=0, Vs=512, Gs=1, V=2000, T=4, H=64, tau=1.0, pm=A16, ytgt=A16, ws=A256,
           wsb=256, hidden=A16):
    binding._tp()
    return L.rlk_linear_logp_fwd_shard(hidden, A16, A16, T, H, V, v0, Vs, tau, pm, A16, A16, Gs,
                                       ytgt, ws, wsb, None)


def _combine(L, nshards=2, Gs=2, V=2000, T=4, pm=A16, ws=A256, wsb=256, lse=A16):
    binding._tp()
    return L.rlk_linear_logp_combine(pm, A16, A16, nshards, Gs, A16, A16, T, V, A16, A16, lse, ws,
                                     wsb, None)


def test_tp_argument_errors(L):
    assert L.rlk_fwd_split_width() == 512
    assert _shard(L, v0=100) == SHAPE              # shard off a split boundary
    assert _shard(L, v0=1536, Vs=512) == INVALID   # past V = 2000
    assert _shard(L, Vs=0) == INVALID
    assert _shard(L, v0=-512) == INVALID
    assert _shard(L, Vs=1024, Gs=1) == INVALID     # row stride below the shard's splits
    assert _shard(L, Gs=5) == INVALID              # row stride above the vocab's splits
    assert _shard(L, H=96) == SHAPE
    assert _shard(L, tau=0.0) == INVALID
    assert _shard(L, T=0, hidden=None) == OK
    assert _shard(L, hidden=None) == INVALID
    assert _shard(L, pm=A16 + 2) == MISALIGNED
    assert _shard(L, wsb=255) == WS_SMALL
    # (nshards - 1) * Gs < ceil(V / 512) <= nshards * Gs
    assert _combine(L, nshards=1, Gs=3) == INVALID
    assert _combine(L, nshards=3, Gs=2) == INVALID
    assert _combine(L, nshards=0) == INVALID
    assert _combine(L, lse=None) == INVALID
    assert _combine(L, pm=A16 + 1) == MISALIGNED
    assert _combine(L, ws=A256 + 8) == MISALIGNED
    assert _combine(L, wsb=100) == WS_SMALL
    assert _combine(L, T=0) == OK


def _bshard(L, v0=0, Vs=8192, V=20000, T=4, H=64, R=4, cps=2, dW=A16, parts=A16, ws=A256,
            wsb=1 << 30, hidden=A16):
    binding._tp()
    return L.rlk_linear_logp_bwd_shard(hidden, A16, A16, T, H, V, v0, Vs, 1.0, A16, A16, A16, A16,
                                       parts, R, cps, dW, ws, wsb, None)


def test_tp_backward_argument_errors(L):
    binding._tp()
    assert L.rlk_bwd_chunk_width(20000) == 8192
    assert L.rlk_bwd_chunk_width(1537) == 1792
    assert L.rlk_bwd_chunk_width(0) == 0
    assert _bshard(L, v0=512) == SHAPE               # off the 8192-row chunk grid
    assert _bshard(L, Vs=9000) == SHAPE              # not the last shard, not whole chunks
    assert _bshard(L, v0=16384, Vs=3616, cps=1) != SHAPE   # the ragged last shard is fine
    assert _bshard(L, v0=16384, Vs=8192) == INVALID  # past V
    assert _bshard(L, R=0) == INVALID
    assert _bshard(L, Vs=16384, cps=1) == INVALID    # fewer slots than the shard's chunks
    assert _bshard(L, cps=4) == INVALID              # more slots than the head has chunks
    assert _bshard(L, dW=None) == INVALID
    assert _bshard(L, dW=A16 + 4) == MISALIGNED
    assert _bshard(L, parts=None) == INVALID
    assert _bshard(L, parts=A16 + 8) == MISALIGNED
    assert _bshard(L, H=96) == SHAPE
    need = binding.workspace_bytes(4, 64, 20000, True)
    assert _bshard(L, wsb=need - 1) == WS_SMALL
    c = L.rlk_dhidden_combine
    assert c(A16, 0, 8, A16, None) == INVALID
    assert c(A16, 2, 6, A16, None) == SHAPE
    assert c(A16, 2, 0, A16, None) == OK
    assert c(None, 2, 8, A16, None) == INVALID
    assert c(A16 + 4, 2, 8, A16, None) == MISALIGNED
    assert c(A16, 2, 8, A16 + 2, None) == MISALIGNED


def test_transition_argument_errors(L):
    binding._tr()
    S = L.rlk_transition_sample
    need = L.rlk_transition_workspace_bytes(3, 24672)
    assert need > 256 and L.rlk_transition_workspace_bytes(-1, 4) == 0

    def smp(B=3, n=24672, x=A16, prev=A16, ws=A256, wsb=need, mean=A16):
        return S(x, A16, A16, A16, A16, A16, B, n, mean, prev, A16, ws, wsb, None)

    assert smp(n=6) == SHAPE                  # n % 4
    assert smp(B=70000) == SHAPE
    assert smp(n=(1 << 24) + 4) == SHAPE
    assert smp(B=-1) == INVALID
    assert smp(B=0, x=None) == OK             # empty: no-op
    assert smp(x=None) == INVALID
    assert smp(prev=None) == INVALID          # sampling writes prev
    assert smp(mean=None) != INVALID          # the mean output is optional
    assert smp(x=A16 + 4) == MISALIGNED
    assert smp(ws=A256 + 16) == MISALIGNED
    assert smp(wsb=need - 1) == WS_SMALL
    lg = L.rlk_transition_logp
    assert lg(A16, A16, None, A16, A16, A16, 3, 24672, None, A16, A256, need, None) == INVALID
    assert lg(A16, A16, A16, A16, A16, A16, 3, 10, None, A16, A256, need, None) == SHAPE


def test_stall_hook_rejects_limits_outside_its_range(L):
    """The fail-closed test hook checks its wait bound (1 ms .. 2 s) before
    anything touches the device: these pointers are never dereferenced."""
    f = L.rlk_test_linear_logp_bwd_stall
    f.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64] * 3 + [ctypes.c_float] + \
        [ctypes.c_void_p] * 7 + [ctypes.c_size_t, ctypes.c_uint64, ctypes.c_int,
                                 ctypes.c_void_p, ctypes.c_uint32, ctypes.c_void_p]
    f.restype = ctypes.c_int
    p = 0x10000
    args = [p, p, p, 4, 64, 100, 1.0, p, p, p, p, p, p, p, 1 << 20]
    assert f(*args, 10, 1, None, 0, None) == INVALID               # below 1 ms
    assert f(*args, 3_000_000_000, 1, None, 0, None) == INVALID    # above 2 s
    assert f(p, p, p, 0, 64, 100, 1.0, p, p, p, p, p, p, p, 1 << 20, 100_000_000, 1,
             None, 0, None) == INVALID                              # T = 0
    assert f(*args, 100_000_000, 1, p, 0, None) == INVALID         # words without seq


def test_forward_stall_hook_checks_its_arguments_first(L):
    """The short-batch forward's test hook rejects T outside 1 .. 256 and limits
    outside 1 ms .. 2 s before anything touches the device: these pointers are
    never dereferenced."""
    f = L.rlk_test_linear_logp_fwd_stall
    f.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64] * 3 + [ctypes.c_float] + \
        [ctypes.c_void_p] * 4 + [ctypes.c_size_t, ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p]
    f.restype = ctypes.c_int
    p = 0x10000
    ok_limit = 100_000_000
    assert f(p, p, p, 4, 64, 100, 1.0, p, p, p, p, 1 << 20, 10, 1, None) == INVALID
    assert f(p, p, p, 4, 64, 100, 1.0, p, p, p, p, 1 << 20, 3_000_000_000, 1, None) == INVALID
    assert f(p, p, p, 0, 64, 100, 1.0, p, p, p, p, 1 << 20, ok_limit, 1, None) == INVALID
    assert f(p, p, p, 257, 64, 100, 1.0, p, p, p, p, 1 << 20, ok_limit, 1, None) == INVALID
    assert f(p, p, p, 4, 64, 100, 1.0, None, p, p, p, 1 << 20, ok_limit, 1, None) == INVALID
