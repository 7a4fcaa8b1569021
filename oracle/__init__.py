"""fp64 CPU oracle for the linear-logp operator -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product (the CUDA library under
``invariant_lm_head_gemm_b200``) never imports it and shares no code with it.

``rlk_oracle.c`` is the oracle proper (plain C, OpenMP over rows/vocab, fp64,
two-pass softmax); ``brute.py`` is an independent dense numpy float64 brute
force used to pin it on tiny inputs.  ``transition.py`` is the fp64 numpy
oracle of the diffusion transition step (pinned by
tests/test_transition_oracle.py).  See the header of ``rlk_oracle.c`` for
the definition each step follows and the passages it rests on.

Pinned by tests/test_oracle_pins.py: brute force on tiny inputs, the uniform
closed form (logp = -ln V, entropy = ln V), the one-hot-dominant limit, the
two-token logistic closed form, invariants (sum p = 1, 0 <= entropy <= ln V,
logp <= 0, max z <= lse <= max z + ln V), vocab-shift invariance, the
temperature identity, central finite differences of the gradient, the
row-sum identity of dz and the uniform-case gradient closed form.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rlk_oracle.c")
_LIB = os.path.join(_HERE, "librlk_oracle.so")
_lib = None

_P = ctypes.c_void_p
_I64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math, no FMA
    contraction) into oracle/librlk_oracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                               "-shared", "-fPIC", "-std=c11", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.rlk_oracle_logits.argtypes = [_P, _P, _I64, _I64, _I64, ctypes.c_double, _P]
        L.rlk_oracle_softmax_stats.argtypes = [_P, _I64, _I64, _P, _P, _P, _P]
        L.rlk_oracle_dlogits.argtypes = [_P, _I64, _I64, _P, ctypes.c_double, _P, _P, _P]
        L.rlk_oracle_dhidden.argtypes = [_P, _P, _I64, _I64, _I64, _P]
        L.rlk_oracle_dw_accumulate.argtypes = [_P, _P, _I64, _I64, _I64, _P]
        L.rlk_oracle_forward.argtypes = [_P, _P, _P, _I64, _I64, _I64, ctypes.c_double,
                                         _P, _P, _P]
        L.rlk_oracle_backward.argtypes = [_P, _P, _P, _I64, _I64, _I64, ctypes.c_double,
                                          _P, _P, _P, _P]
        L.rlk_oracle_set_mutation.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a):
    return np.ascontiguousarray(a, dtype=np.uint16)


def _check(rc, what):
    if rc != 0:
        raise ValueError("oracle %s failed with code %d" % (what, rc))


def tau_of(temperature) -> float:
    """The temperature as the operator receives it: an fp32 value, widened."""
    return float(np.float32(temperature))


def logits(hidden, W, temperature):
    """z[T,V] = (hidden . W^T) / tau in fp64 (steps 1-2)."""
    hidden, W = _u16(hidden), _u16(W)
    T, H = hidden.shape
    V = W.shape[0]
    z = np.empty((T, V), np.float64)
    _check(lib().rlk_oracle_logits(_ptr(hidden), _ptr(W), T, H, V, tau_of(temperature), _ptr(z)),
           "logits")
    return z


def softmax_stats(z, targets):
    """(logp, entropy, lse) per row from dense z (steps 3-4)."""
    z = np.ascontiguousarray(z, np.float64)
    targets = np.ascontiguousarray(targets, np.int64)
    T, V = z.shape
    out = [np.empty(T, np.float64) for _ in range(3)]
    _check(lib().rlk_oracle_softmax_stats(_ptr(z), T, V, _ptr(targets), *map(_ptr, out)),
           "softmax_stats")
    return tuple(out)


def dlogits(z, targets, temperature, dlogp, dentropy):
    """dx[T,V] = dz / tau (step 5)."""
    z = np.ascontiguousarray(z, np.float64)
    targets = np.ascontiguousarray(targets, np.int64)
    dl = np.ascontiguousarray(dlogp, np.float64)
    de = np.ascontiguousarray(dentropy, np.float64)
    T, V = z.shape
    dx = np.empty((T, V), np.float64)
    _check(lib().rlk_oracle_dlogits(_ptr(z), T, V, _ptr(targets), tau_of(temperature),
                                    _ptr(dl), _ptr(de), _ptr(dx)), "dlogits")
    return dx


def dhidden(dx, W):
    """dHidden[T,H] = dx . W (step 6a)."""
    dx = np.ascontiguousarray(dx, np.float64)
    W = _u16(W)
    T, V = dx.shape
    H = W.shape[1]
    out = np.empty((T, H), np.float64)
    _check(lib().rlk_oracle_dhidden(_ptr(dx), _ptr(W), T, H, V, _ptr(out)), "dhidden")
    return out


def dw(dx, hidden):
    """dW[V,H] = dx^T . hidden (step 6b)."""
    dx = np.ascontiguousarray(dx, np.float64)
    hidden = _u16(hidden)
    T, V = dx.shape
    H = hidden.shape[1]
    out = np.zeros((V, H), np.float64)
    _check(lib().rlk_oracle_dw_accumulate(_ptr(dx), _ptr(hidden), T, H, V, _ptr(out)), "dw")
    return out


def forward(hidden, W, targets, temperature):
    """(logp, entropy, lse) fp64 for every row, streaming 64-row blocks."""
    hidden, W = _u16(hidden), _u16(W)
    targets = np.ascontiguousarray(targets, np.int64)
    T, H = hidden.shape
    V = W.shape[0]
    out = [np.empty(T, np.float64) for _ in range(3)]
    _check(lib().rlk_oracle_forward(_ptr(hidden), _ptr(W), _ptr(targets), T, H, V,
                                    tau_of(temperature), *map(_ptr, out)), "forward")
    return tuple(out)


def backward(hidden, W, targets, temperature, dlogp, dentropy):
    """(dHidden[T,H], dW[V,H]) fp64, streaming 64-row blocks."""
    hidden, W = _u16(hidden), _u16(W)
    targets = np.ascontiguousarray(targets, np.int64)
    dl = np.ascontiguousarray(dlogp, np.float64)
    de = np.ascontiguousarray(dentropy, np.float64)
    T, H = hidden.shape
    V = W.shape[0]
    dH = np.empty((T, H), np.float64)
    dWo = np.empty((V, H), np.float64)
    _check(lib().rlk_oracle_backward(_ptr(hidden), _ptr(W), _ptr(targets), T, H, V,
                                     tau_of(temperature), _ptr(dl), _ptr(de), _ptr(dH),
                                     _ptr(dWo)), "backward")
    return dH, dWo


def num_threads() -> int:
    return int(lib().rlk_oracle_num_threads())


class mutation:
    """Context manager that plants one known mistake in the oracle (tests
    only).  Codes are listed in rlk_oracle.c."""

    NAMES = {1: "no_temperature", 2: "entropy_sign", 3: "target_shift", 4: "lse_no_max",
             5: "dx_no_entropy", 6: "dx_onehot_sign", 7: "dw_row_index", 8: "dx_no_tau",
             9: "ez_is_max", 10: "dot_skip_last", 11: "dh_transposed"}

    def __init__(self, code: int):
        self.code = code

    def __enter__(self):
        _check(lib().rlk_oracle_set_mutation(self.code), "set_mutation")
        return self

    def __exit__(self, *exc):
        lib().rlk_oracle_set_mutation(0)
        return False
