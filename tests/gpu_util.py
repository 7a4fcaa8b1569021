"""Helpers shared by the GPU tests: moving seeded inputs to the device,
running the library through its C ABI, and the parity tolerances.

Tolerances (the linear-logp target statement): |d logp| and |d entropy|
(and |d lse|) <= 2e-3 + 1e-3 |ref|; dHidden and dW relative Frobenius error
<= 5e-3 against the fp64 oracle."""
from __future__ import annotations

import numpy as np
import torch

from invariant_lm_head_gemm_b200 import binding
from invariant_lm_head_gemm_b200 import workloads as wl

ABS_TOL = 2e-3
REL_TOL = 1e-3
FROB_TOL = 5e-3


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def dev(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dtype).cuda()


def run(hidden_bits, W_dev, targets, tau, dlogp=None, dentropy=None, ws=None, hidden_dev=None):
    """Forward (and backward when dlogp is given) through the C ABI.  Returns
    a dict of device tensors and the device error word."""
    T, H = hidden_bits.shape if hidden_dev is None else hidden_dev.shape
    V = W_dev.shape[0]
    hid = hidden_dev if hidden_dev is not None else dev_bf16(hidden_bits)
    tg = dev(targets, torch.int64)
    if ws is None:
        ws = binding.make_workspace(T, H, V, True)
    logp, ent, lse = binding.rlk_linear_logp_fwd(hid, W_dev, tg, tau, ws)
    out = dict(logp=logp, entropy=ent, lse=lse)
    if dlogp is not None:
        dH, dW = binding.rlk_linear_logp_bwd(hid, W_dev, tg, tau, lse, ent,
                                             dev(dlogp, torch.float32),
                                             dev(dentropy, torch.float32), ws)
        out.update(dH=dH, dW=dW)
    torch.cuda.synchronize()
    out["err"] = binding.rlk_read_device_error(ws)
    return out


def assert_close_vec(got, ref, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    tol = ABS_TOL + REL_TOL * np.abs(ref)
    bad = np.abs(got - ref) > tol
    assert not bad.any(), "%s: %d/%d outside tolerance; worst |d|=%.3g at %d (got %r ref %r)" % (
        what, int(bad.sum()), bad.size, float(np.max(np.abs(got - ref))),
        int(np.argmax(np.abs(got - ref))), got[np.argmax(np.abs(got - ref))],
        ref[np.argmax(np.abs(got - ref))])
    return float(np.max(np.abs(got - ref)))


def rel_frob(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def random_case(T, H, V, tau, seed, wstd=0.05):
    """Seeded rows + W of arbitrary shape (edge-case parity); targets include
    the first and last vocab entries."""
    hidden, targets = wl.make_rows(seed, T, H, V)
    W = wl.make_weight(seed, V, H, std=wstd)
    targets[0] = 0
    targets[-1] = V - 1
    rng = np.random.default_rng(seed + 1000)
    dlogp = rng.standard_normal(T).astype(np.float32)
    dent = (0.1 * rng.standard_normal(T)).astype(np.float32)
    return wl.Workload("case", T, H, V, tau, hidden, W, targets, dlogp, dent, seed=seed)
