"""Dense numpy float64 brute force of the linear-logp operator -- TEST
INFRASTRUCTURE ONLY (pins the C oracle on tiny inputs).

It deliberately takes textbook routes that differ from the C oracle's:
  * the softmax is formed explicitly as p = exp(z - max) / sum(exp(z - max));
  * logp = log(p[target]) and entropy = -sum p log p (Shannon, nats);
  * the gradient goes through the explicit softmax Jacobian
    J = diag(p) - p p^T:  d logp/dz = e_target - p and
    d entropy/dz = -J (log p + 1);
  * dHidden and dW are numpy matmuls of the dense dlogits.
Only for shapes where a dense [V,V] Jacobian per row fits in memory.
"""
from __future__ import annotations

import numpy as np


def _widen(bits):
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def forward(hidden_bits, W_bits, targets, temperature):
    tau = float(np.float32(temperature))
    h = _widen(hidden_bits)
    w = _widen(W_bits)
    z = (h @ w.T) / tau
    e = np.exp(z - z.max(axis=1, keepdims=True))
    p = e / e.sum(axis=1, keepdims=True)
    rows = np.arange(z.shape[0])
    logp = np.log(p[rows, targets])
    with np.errstate(divide="ignore", invalid="ignore"):
        plogp = np.where(p > 0, p * np.log(p), 0.0)
    entropy = -plogp.sum(axis=1)
    lse = z[rows, targets] - logp
    return logp, entropy, lse, z, p


def backward(hidden_bits, W_bits, targets, temperature, dlogp, dentropy):
    tau = float(np.float32(temperature))
    h = _widen(hidden_bits)
    w = _widen(W_bits)
    _, _, _, z, p = forward(hidden_bits, W_bits, targets, temperature)
    T, V = z.shape
    dz = np.empty_like(z)
    for t in range(T):
        pt = p[t]
        J = np.diag(pt) - np.outer(pt, pt)
        g_logp = -pt.copy()
        g_logp[targets[t]] += 1.0
        g_ent = -J @ (np.log(pt) + 1.0)
        dz[t] = float(dlogp[t]) * g_logp + float(dentropy[t]) * g_ent
    dx = dz / tau
    return dx @ w, dx.T @ h, dx
