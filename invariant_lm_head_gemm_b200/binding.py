"""Thin Python binding of librlk.so (include/rlk.h) for torch tensors.

Argument marshalling only: every step of the operator runs in the library's
CUDA kernels.  There is no fallback; if the library is missing or the device
is not a B200 the calls raise.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librlk.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "rlk.h")

RLK_DEVERR_TARGET = 0x1
RLK_DEVERR_TIMEOUT = 0x2

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_lib = None


class RlkError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s failed: %s" % (what, status_string(status)))


def lib():
    """Load librlk.so (built in-tree by ``python -m invariant_lm_head_gemm_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("librlk.so is not built (%s); run "
                               "`python -m invariant_lm_head_gemm_b200.build`" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        L.rlk_linear_logp_workspace_bytes.argtypes = [_I64, _I64, _I64, ctypes.c_int]
        L.rlk_linear_logp_workspace_bytes.restype = ctypes.c_size_t
        L.rlk_linear_logp_fwd.argtypes = [_P, _P, _P, _I64, _I64, _I64, ctypes.c_float,
                                          _P, _P, _P, _P, ctypes.c_size_t, _P]
        L.rlk_linear_logp_fwd.restype = ctypes.c_int
        L.rlk_linear_logp_bwd.argtypes = [_P, _P, _P, _I64, _I64, _I64, ctypes.c_float,
                                          _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
        L.rlk_linear_logp_bwd.restype = ctypes.c_int
        L.rlk_gemm_workspace_bytes.argtypes = []
        L.rlk_gemm_workspace_bytes.restype = ctypes.c_size_t
        L.rlk_gemm_bf16_f32.argtypes = [_P, _P, _I64, _I64, _I64, ctypes.c_int, ctypes.c_int,
                                        _P, _P, ctypes.c_size_t, _P]
        L.rlk_gemm_bf16_f32.restype = ctypes.c_int
        L.rlk_backend_id.argtypes = []
        L.rlk_backend_id.restype = ctypes.c_char_p
        L.rlk_call_count.argtypes = [ctypes.c_int]
        L.rlk_call_count.restype = ctypes.c_uint64
        L.rlk_read_device_error.argtypes = [_P, ctypes.POINTER(ctypes.c_uint32), _P]
        L.rlk_read_device_error.restype = ctypes.c_int
        L.rlk_status_string.argtypes = [ctypes.c_int]
        L.rlk_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def declared_functions():
    """Names of the functions declared in include/rlk.h."""
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rlk_[a-z0-9_]+)\s*\(", text)))


def status_string(status: int) -> str:
    return lib().rlk_status_string(int(status)).decode()


def backend_id() -> str:
    return lib().rlk_backend_id().decode()


def call_count(which: int) -> int:
    return int(lib().rlk_call_count(which))


def _check(status, what):
    if status != 0:
        raise RlkError(status, what)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def workspace_bytes(T: int, H: int, V: int, for_backward: bool = True) -> int:
    return int(lib().rlk_linear_logp_workspace_bytes(T, H, V, 1 if for_backward else 0))


def make_workspace(T: int, H: int, V: int, for_backward: bool = True, device=None):
    """A zeroed workspace tensor (uint8) big enough for these sizes."""
    n = workspace_bytes(T, H, V, for_backward)
    if n == 0:
        raise ValueError("unsupported sizes T=%d H=%d V=%d" % (T, H, V))
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def _req(t, dtype, name, ndim):
    if t.dtype != dtype or not t.is_cuda or not t.is_contiguous() or t.dim() != ndim:
        raise ValueError("%s must be a contiguous CUDA %s tensor with %d dims" % (name, dtype, ndim))


def rlk_linear_logp_fwd(hidden, W, targets, temperature, workspace=None, out=None, stream=None):
    """logp, entropy, lse [T] fp32 of hidden [T,H] bf16 against W [V,H] bf16."""
    _req(hidden, torch.bfloat16, "hidden", 2)
    _req(W, torch.bfloat16, "W", 2)
    _req(targets, torch.int64, "targets", 1)
    T, H = hidden.shape
    V = W.shape[0]
    if W.shape[1] != H or targets.shape[0] != T:
        raise ValueError("shape mismatch")
    if workspace is None:
        workspace = make_workspace(T, H, V, False, hidden.device)
    if out is None:
        out = tuple(torch.empty(T, dtype=torch.float32, device=hidden.device) for _ in range(3))
    logp, entropy, lse = out
    _check(lib().rlk_linear_logp_fwd(_ptr(hidden), _ptr(W), _ptr(targets), T, H, V,
                                     float(temperature), _ptr(logp), _ptr(entropy), _ptr(lse),
                                     _ptr(workspace), workspace.numel(), _stream(stream)),
           "rlk_linear_logp_fwd")
    return logp, entropy, lse


def rlk_linear_logp_bwd(hidden, W, targets, temperature, lse, entropy, dlogp, dentropy,
                        workspace=None, out=None, stream=None):
    """dHidden [T,H] bf16 and dW [V,H] fp32 (both overwritten)."""
    _req(hidden, torch.bfloat16, "hidden", 2)
    _req(W, torch.bfloat16, "W", 2)
    _req(targets, torch.int64, "targets", 1)
    for n, t in (("lse", lse), ("entropy", entropy), ("dlogp", dlogp), ("dentropy", dentropy)):
        _req(t, torch.float32, n, 1)
    T, H = hidden.shape
    V = W.shape[0]
    if workspace is None:
        workspace = make_workspace(T, H, V, True, hidden.device)
    if out is None:
        out = (torch.empty(T, H, dtype=torch.bfloat16, device=hidden.device),
               torch.empty(V, H, dtype=torch.float32, device=hidden.device))
    dHidden, dW = out
    _check(lib().rlk_linear_logp_bwd(_ptr(hidden), _ptr(W), _ptr(targets), T, H, V,
                                     float(temperature), _ptr(lse), _ptr(entropy), _ptr(dlogp),
                                     _ptr(dentropy), _ptr(dHidden), _ptr(dW), _ptr(workspace),
                                     workspace.numel(), _stream(stream)),
           "rlk_linear_logp_bwd")
    return dHidden, dW


_signal_fns = None


def _signal():
    global _signal_fns
    if _signal_fns is None:
        L = lib()
        f = L.rlk_linear_logp_bwd_signal
        f.argtypes = [_P, _P, _P, _I64, _I64, _I64, ctypes.c_float, _P, _P, _P, _P, _P, _P, _P,
                      ctypes.c_size_t, _P, ctypes.c_uint32, _P]
        f.restype = ctypes.c_int
        w = L.rlk_stream_wait_chunk
        w.argtypes = [_P, ctypes.c_uint32, _P]
        w.restype = ctypes.c_int
        _signal_fns = (f, w)
    return _signal_fns


def rlk_linear_logp_bwd_signal(hidden, W, targets, temperature, lse, entropy, dlogp, dentropy,
                               workspace, out, chunk_done, seq, stream=None):
    """rlk_linear_logp_bwd that also sets chunk_done[c] (int32 device words, one
    per vocab chunk of rlk_bwd_chunk_width(V) rows) to seq once chunk c's dW
    rows are written."""
    T, H = hidden.shape
    V = W.shape[0]
    dHidden, dW = out
    if chunk_done.dtype != torch.int32 or not chunk_done.is_cuda or \
            chunk_done.numel() < -(-V // bwd_chunk_width(V)):
        raise ValueError("chunk_done: int32 CUDA tensor with one word per vocab chunk")
    _check(_signal()[0](_ptr(hidden), _ptr(W), _ptr(targets), T, H, V, float(temperature),
                        _ptr(lse), _ptr(entropy), _ptr(dlogp), _ptr(dentropy), _ptr(dHidden),
                        _ptr(dW), _ptr(workspace), workspace.numel(), _ptr(chunk_done), int(seq),
                        _stream(stream)),
           "rlk_linear_logp_bwd_signal")
    return dHidden, dW


def rlk_stream_wait_chunk(chunk_word, seq, stream=None):
    """Makes `stream` wait on the device until chunk_word (a one-element int32
    CUDA tensor view) holds seq or more."""
    _check(_signal()[1](_ptr(chunk_word), int(seq), _stream(stream)), "rlk_stream_wait_chunk")


_stall_fn = None


def rlk_test_linear_logp_bwd_stall(hidden, W, targets, temperature, lse, entropy, dlogp,
                                   dentropy, workspace, out, wait_limit_ns, stall,
                                   chunk_done=None, seq=0, stream=None):
    """Test hook of the fail-closed path: the backward with every wait bounded
    by wait_limit_ns and, when stall is set, one dependency that is never met
    (the device error word then reports RLK_DEVERR_TIMEOUT)."""
    global _stall_fn
    if _stall_fn is None:
        f = lib().rlk_test_linear_logp_bwd_stall
        f.argtypes = [_P, _P, _P, _I64, _I64, _I64, ctypes.c_float, _P, _P, _P, _P, _P, _P, _P,
                      ctypes.c_size_t, ctypes.c_uint64, ctypes.c_int, _P, ctypes.c_uint32, _P]
        f.restype = ctypes.c_int
        _stall_fn = f
    T, H = hidden.shape
    V = W.shape[0]
    dHidden, dW = out
    _check(_stall_fn(_ptr(hidden), _ptr(W), _ptr(targets), T, H, V, float(temperature), _ptr(lse),
                     _ptr(entropy), _ptr(dlogp), _ptr(dentropy), _ptr(dHidden), _ptr(dW),
                     _ptr(workspace), workspace.numel(), int(wait_limit_ns), int(stall),
                     _ptr(chunk_done), int(seq), _stream(stream)),
           "rlk_test_linear_logp_bwd_stall")
    return dHidden, dW


_fwd_stall_fn = None


def rlk_test_linear_logp_fwd_stall(hidden, W, targets, temperature, workspace, out, wait_limit_ns,
                                   stall, stream=None):
    """Test hook of the short-batch forward's fail-closed path (T <= 256): every
    wait bounded by wait_limit_ns and, when stall is set, one accumulator that
    never reports full (the device error word then reports
    RLK_DEVERR_TIMEOUT)."""
    global _fwd_stall_fn
    if _fwd_stall_fn is None:
        f = lib().rlk_test_linear_logp_fwd_stall
        f.argtypes = [_P, _P, _P, _I64, _I64, _I64, ctypes.c_float, _P, _P, _P, _P,
                      ctypes.c_size_t, ctypes.c_uint64, ctypes.c_int, _P]
        f.restype = ctypes.c_int
        _fwd_stall_fn = f
    T, H = hidden.shape
    V = W.shape[0]
    logp, entropy, lse = out
    _check(_fwd_stall_fn(_ptr(hidden), _ptr(W), _ptr(targets), T, H, V, float(temperature),
                         _ptr(logp), _ptr(entropy), _ptr(lse), _ptr(workspace), workspace.numel(),
                         int(wait_limit_ns), int(stall), _stream(stream)),
           "rlk_test_linear_logp_fwd_stall")
    return logp, entropy, lse


def rlk_gemm_bf16_f32(A, B, a_mn_major=False, b_mn_major=False, stream=None, out=None,
                      workspace=None):
    """C = A' . B'^T through the tensor-core mainloop (self-check entry).
    A' is A ([M,K]) or A^T (A stored [K,M] when a_mn_major); B' likewise.
    `out` (fp32 [M,N]) and `workspace` (zeroed uint8, rlk_gemm_workspace_bytes
    long) may be given to reuse buffers across calls."""
    _req(A, torch.bfloat16, "A", 2)
    _req(B, torch.bfloat16, "B", 2)
    M, K = (A.shape[1], A.shape[0]) if a_mn_major else A.shape
    N, K2 = (B.shape[1], B.shape[0]) if b_mn_major else B.shape
    if K != K2:
        raise ValueError("K mismatch")
    if out is None:
        C = torch.empty(M, N, dtype=torch.float32, device=A.device)
    else:
        _req(out, torch.float32, "out", 2)
        if tuple(out.shape) != (M, N):
            raise ValueError("out must be [M, N]")
        C = out
    if workspace is None:
        ws = torch.zeros(int(lib().rlk_gemm_workspace_bytes()), dtype=torch.uint8,
                         device=A.device)
    else:
        ws = workspace
    _check(lib().rlk_gemm_bf16_f32(_ptr(A), _ptr(B), M, N, K, int(a_mn_major), int(b_mn_major),
                                   _ptr(C), _ptr(ws), ws.numel(), _stream(stream)),
           "rlk_gemm_bf16_f32")
    return C, ws


def rlk_read_device_error(workspace, stream=None) -> int:
    """RLK_DEVERR_* bits recorded in the workspace (then cleared).  Syncs."""
    v = ctypes.c_uint32(0)
    _check(lib().rlk_read_device_error(_ptr(workspace), ctypes.byref(v), _stream(stream)),
           "rlk_read_device_error")
    return int(v.value)


class LinearLogp(torch.autograd.Function):
    """autograd wrapper: (logp, entropy) = LinearLogp.apply(hidden, W, targets, temperature).
    Gradients flow to hidden (bf16) and W (fp32 cast to W's dtype)."""

    @staticmethod
    def forward(ctx, hidden, W, targets, temperature):
        T, H = hidden.shape
        ws = make_workspace(T, H, W.shape[0], True, hidden.device)
        logp, entropy, lse = rlk_linear_logp_fwd(hidden, W, targets, temperature, ws)
        ctx.save_for_backward(hidden, W, targets, lse, entropy)
        ctx.temperature = temperature
        ctx.ws = ws
        return logp, entropy

    @staticmethod
    def backward(ctx, dlogp, dentropy):
        hidden, W, targets, lse, entropy = ctx.saved_tensors
        T = hidden.shape[0]
        dl = (dlogp if dlogp is not None else torch.zeros(T, device=hidden.device)).float()
        de = (dentropy if dentropy is not None else torch.zeros(T, device=hidden.device)).float()
        dH, dW = rlk_linear_logp_bwd(hidden, W, targets, ctx.temperature, lse, entropy,
                                     dl.contiguous(), de.contiguous(), ctx.ws)
        return dH, dW.to(W.dtype), None, None


_noalloc_fn = None


def rlk_linear_logp_fwd_noalloc(hidden, W, targets, temperature, out=None, stream=None):
    """Forward through the entry point that takes no workspace and allocates
    nothing (its scratch is a fixed device array inside the library); for
    callers that cannot allocate device memory.  Outputs as rlk_linear_logp_fwd."""
    global _noalloc_fn
    if _noalloc_fn is None:
        f = lib().rlk_linear_logp_fwd_noalloc
        f.argtypes = [_P, _P, _P, _I64, _I64, _I64, ctypes.c_float, _P, _P, _P, _P]
        f.restype = ctypes.c_int
        _noalloc_fn = f
    _req(hidden, torch.bfloat16, "hidden", 2)
    _req(W, torch.bfloat16, "W", 2)
    _req(targets, torch.int64, "targets", 1)
    T, H = hidden.shape
    V = W.shape[0]
    if W.shape[1] != H or targets.shape[0] != T:
        raise ValueError("shape mismatch")
    if out is None:
        out = tuple(torch.empty(T, dtype=torch.float32, device=hidden.device) for _ in range(3))
    logp, entropy, lse = out
    _check(_noalloc_fn(_ptr(hidden), _ptr(W), _ptr(targets), T, H, V, float(temperature),
                       _ptr(logp), _ptr(entropy), _ptr(lse), _stream(stream)),
           "rlk_linear_logp_fwd_noalloc")
    return logp, entropy, lse


_sum_fn = None


def rlk_sum_ordered(parts, out=None, stream=None):
    """out = ((parts[0] + parts[1]) + parts[2]) + ... elementwise in fp32, in
    list order (1..64 equally shaped contiguous CUDA fp32 tensors)."""
    global _sum_fn
    if _sum_fn is None:
        f = lib().rlk_sum_ordered
        f.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int, _P, _I64, _P]
        f.restype = ctypes.c_int
        _sum_fn = f
    n = parts[0].numel()
    for t in parts:
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or t.numel() != n:
            raise ValueError("parts must be contiguous CUDA fp32 tensors of equal size")
    if out is None:
        out = torch.empty_like(parts[0])
    arr = (ctypes.c_void_p * len(parts))(*[t.data_ptr() for t in parts])
    _check(_sum_fn(arr, len(parts), _ptr(out), n, _stream(stream)), "rlk_sum_ordered")
    return out


_tp_fns = None


def _tp():
    global _tp_fns
    if _tp_fns is None:
        L = lib()
        L.rlk_fwd_split_width.argtypes = []
        L.rlk_fwd_split_width.restype = ctypes.c_int64
        L.rlk_linear_logp_fwd_shard.argtypes = [_P, _P, _P, _I64, _I64, _I64, _I64, _I64,
                                                ctypes.c_float, _P, _P, _P, _I64, _P, _P,
                                                ctypes.c_size_t, _P]
        L.rlk_linear_logp_fwd_shard.restype = ctypes.c_int
        L.rlk_linear_logp_combine.argtypes = [_P, _P, _P, _I64, _I64, _P, _P, _I64, _I64, _P, _P,
                                              _P, _P, ctypes.c_size_t, _P]
        L.rlk_linear_logp_combine.restype = ctypes.c_int
        L.rlk_bwd_chunk_width.argtypes = [_I64]
        L.rlk_bwd_chunk_width.restype = ctypes.c_int64
        L.rlk_linear_logp_bwd_shard.argtypes = [_P, _P, _P, _I64, _I64, _I64, _I64, _I64,
                                                ctypes.c_float, _P, _P, _P, _P, _P, _I64, _I64,
                                                _P, _P, ctypes.c_size_t, _P]
        L.rlk_linear_logp_bwd_shard.restype = ctypes.c_int
        L.rlk_dhidden_combine.argtypes = [_P, _I64, _I64, _P, _P]
        L.rlk_dhidden_combine.restype = ctypes.c_int
        _tp_fns = L
    return _tp_fns


def fwd_split_width() -> int:
    """Vocab columns per forward split (shards must start at multiples of it)."""
    return int(_tp().rlk_fwd_split_width())


def rlk_linear_logp_fwd_shard(hidden, W_shard, targets, V, v0, temperature, part, ytgt,
                              workspace=None, stream=None):
    """Split triples of one vocab shard.  part: (part_m, part_s, part_b), each a
    contiguous fp32 [T, Gs] tensor (Gs the same on every shard); ytgt: fp32 [T]
    (rows with targets in the shard are written)."""
    _req(hidden, torch.bfloat16, "hidden", 2)
    _req(W_shard, torch.bfloat16, "W_shard", 2)
    _req(targets, torch.int64, "targets", 1)
    T, H = hidden.shape
    if workspace is None:
        workspace = torch.zeros(256, dtype=torch.uint8, device=hidden.device)
    pm, ps, pb = part
    for p in part:
        _req(p, torch.float32, "part", 2)
        if p.shape != pm.shape or p.shape[0] != T:
            raise ValueError("part buffers must all be [T, Gs]")
    _req(ytgt, torch.float32, "ytgt", 1)
    _check(_tp().rlk_linear_logp_fwd_shard(_ptr(hidden), _ptr(W_shard), _ptr(targets), T, H, V,
                                           v0, W_shard.shape[0], float(temperature), _ptr(pm),
                                           _ptr(ps), _ptr(pb), pm.shape[1], _ptr(ytgt),
                                           _ptr(workspace),
                                           workspace.numel(), _stream(stream)),
           "rlk_linear_logp_fwd_shard")
    return workspace


def rlk_linear_logp_combine(part, nshards, Gs, ytgt, targets, V, out=None, workspace=None,
                            stream=None):
    """logp, entropy, lse from split triples laid out [nshards][T][Gs]."""
    T = targets.shape[0]
    dev = targets.device
    if workspace is None:
        workspace = torch.zeros(256, dtype=torch.uint8, device=dev)
    if out is None:
        out = tuple(torch.empty(T, dtype=torch.float32, device=dev) for _ in range(3))
    pm, ps, pb = part
    logp, entropy, lse = out
    _check(_tp().rlk_linear_logp_combine(_ptr(pm), _ptr(ps), _ptr(pb), nshards, Gs, _ptr(ytgt),
                                         _ptr(targets), T, V, _ptr(logp), _ptr(entropy),
                                         _ptr(lse), _ptr(workspace), workspace.numel(),
                                         _stream(stream)),
           "rlk_linear_logp_combine")
    return out


def bwd_chunk_width(V: int) -> int:
    """Vocab rows per backward chunk of a V-row head (shards of the backward
    start at multiples of it)."""
    return int(_tp().rlk_bwd_chunk_width(V))


def rlk_linear_logp_bwd_shard(hidden, W_shard, targets, V, v0, temperature, lse, entropy, dlogp,
                              dentropy, dh_parts, part_rows, dW_shard=None, workspace=None,
                              stream=None):
    """dW rows of one vocab shard and its per-chunk dHidden products.
    dh_parts: contiguous fp32 [S, part_chunks, part_rows, H] (S = ceil(T /
    part_rows)).  Returns (dW_shard, workspace)."""
    _req(hidden, torch.bfloat16, "hidden", 2)
    _req(W_shard, torch.bfloat16, "W_shard", 2)
    _req(targets, torch.int64, "targets", 1)
    _req(dh_parts, torch.float32, "dh_parts", 4)
    T, H = hidden.shape
    S, part_chunks, rows, Hp = dh_parts.shape
    if rows != part_rows or Hp != H or S * part_rows < T:
        raise ValueError("dh_parts must be [ceil(T/part_rows), part_chunks, part_rows, H]")
    if dW_shard is None:
        dW_shard = torch.empty(W_shard.shape[0], H, dtype=torch.float32, device=hidden.device)
    if workspace is None:
        workspace = make_workspace(T, H, V, True, hidden.device)
    _check(_tp().rlk_linear_logp_bwd_shard(_ptr(hidden), _ptr(W_shard), _ptr(targets), T, H, V,
                                           v0, W_shard.shape[0], float(temperature), _ptr(lse),
                                           _ptr(entropy), _ptr(dlogp), _ptr(dentropy),
                                           _ptr(dh_parts), part_rows, part_chunks,
                                           _ptr(dW_shard), _ptr(workspace), workspace.numel(),
                                           _stream(stream)),
           "rlk_linear_logp_bwd_shard")
    return dW_shard, workspace


def rlk_dhidden_combine(dh_parts, nparts, out, stream=None):
    """out (bf16, any shape) = the fixed-order sum of the first nparts blocks of
    dh_parts (fp32, viewed as [blocks, out.numel()])."""
    count = out.numel()
    if not (dh_parts.is_contiguous() and dh_parts.dtype == torch.float32 and out.is_contiguous()
            and out.dtype == torch.bfloat16 and dh_parts.numel() >= nparts * count):
        raise ValueError("dh_parts: contiguous fp32 holding nparts blocks; out: contiguous bf16")
    _check(_tp().rlk_dhidden_combine(_ptr(dh_parts), nparts, count, _ptr(out), _stream(stream)),
           "rlk_dhidden_combine")
    return out


_tr_fns = None


def _tr():
    global _tr_fns
    if _tr_fns is None:
        L = lib()
        L.rlk_transition_workspace_bytes.argtypes = [_I64, _I64]
        L.rlk_transition_workspace_bytes.restype = ctypes.c_size_t
        L.rlk_transition_sample.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I64, _P, _P, _P, _P,
                                            ctypes.c_size_t, _P]
        L.rlk_transition_sample.restype = ctypes.c_int
        L.rlk_transition_logp.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I64, _P, _P, _P,
                                          ctypes.c_size_t, _P]
        L.rlk_transition_logp.restype = ctypes.c_int
        _tr_fns = L
    return _tr_fns


def transition_workspace(B: int, n: int, device=None):
    nbytes = _tr().rlk_transition_workspace_bytes(B, n)
    if nbytes == 0:
        raise ValueError("unsupported sizes B=%d n=%d" % (B, n))
    return torch.zeros(nbytes, dtype=torch.uint8, device=device or "cuda")


def _tr_args(x, v, third, a, c, s):
    for t, name in ((x, "x"), (v, "v"), (third, "eps/prev")):
        _req(t, torch.float32, name, 2)
    for t, name in ((a, "a"), (c, "c"), (s, "s")):
        _req(t, torch.float32, name, 1)
    B, n = x.shape
    if v.shape != x.shape or third.shape != x.shape or a.shape[0] != B or c.shape[0] != B \
            or s.shape[0] != B:
        raise ValueError("x, v, eps/prev must be [B, n]; a, c, s [B]")
    return B, n


def rlk_transition_sample(x, v, eps, a, c, s, want_mean=True, out=None, workspace=None,
                          stream=None):
    """(mean or None, prev, logp) of one sampling step: x, v, eps fp32 [B, n]
    (n = L * D flattened), a, c, s fp32 [B]."""
    B, n = _tr_args(x, v, eps, a, c, s)
    if out is None:
        out = (torch.empty_like(x) if want_mean else None, torch.empty_like(x),
               torch.empty(B, dtype=torch.float32, device=x.device))
    mean, prev, logp = out
    if workspace is None:
        workspace = transition_workspace(B, n, x.device)
    _check(_tr().rlk_transition_sample(_ptr(x), _ptr(v), _ptr(eps), _ptr(a), _ptr(c), _ptr(s), B,
                                       n, _ptr(mean) if mean is not None else None, _ptr(prev),
                                       _ptr(logp), _ptr(workspace), workspace.numel(),
                                       _stream(stream)),
           "rlk_transition_sample")
    return mean, prev, logp


def rlk_transition_logp(x, v, prev, a, c, s, want_mean=False, out=None, workspace=None,
                        stream=None):
    """(mean or None, logp) of scoring a recorded prev_sample."""
    B, n = _tr_args(x, v, prev, a, c, s)
    if out is None:
        out = (torch.empty_like(x) if want_mean else None,
               torch.empty(B, dtype=torch.float32, device=x.device))
    mean, logp = out
    if workspace is None:
        workspace = transition_workspace(B, n, x.device)
    _check(_tr().rlk_transition_logp(_ptr(x), _ptr(v), _ptr(prev), _ptr(a), _ptr(c), _ptr(s), B,
                                     n, _ptr(mean) if mean is not None else None, _ptr(logp),
                                     _ptr(workspace), workspace.numel(), _stream(stream)),
           "rlk_transition_logp")
    return mean, logp
