"""Seeded synthetic inputs for the linear-logp operator.

This module only draws random numbers and rounds them to bf16.  It holds none
of the operator's arithmetic, so both sides of every comparison (the CUDA
library and the fp64 CPU oracle) are fed from here.

Workloads follow the shapes of the RL-Kernel evidence pages:
  * H=4096, V=151936 is the Qwen3-8B LM head that the VIME dense experiment
    page ("Required gates": Qwen3-8B, BF16, temperature 1) runs the bitwise
    linear-logp route on;
  * about 5200 tokens per RL step, 8 samples per step (h100-cp-gradient.json,
    runs[0].tokens."0"/"1": token_count 5208 / 5016, sample_count 8);
  * the batch-invariance probe follows the "batch_invariant" and
    "forward_rows_independent" gates of the h3-runtime-integration-b200
    report (lora_gate / transition blocks).
No dataset or checkpoint is used: DAPO-Math-17k prompts and Qwen3-8B weights
are stood in for by seeded Gaussian draws of the same shapes.

Random streams: each tensor has its own child of ``SeedSequence(seed)`` so
that, e.g., W for a given seed does not depend on T.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

# child-stream indices of SeedSequence(seed).spawn(N_STREAMS)
_S_HIDDEN, _S_W, _S_TARGET, _S_DLOGP, _S_LENGTHS, _S_POS = range(6)
N_STREAMS = 6

W_STD = 0.02
W_BLOCK_ROWS = 4096


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 with round-to-nearest-even, returning the
    16-bit patterns (uint16).  Direct rounding from float64 (no detour through
    float32, which could double-round).  Finite inputs only."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    bits = x.view(np.uint64)
    lsb = (bits >> np.uint64(45)) & np.uint64(1)
    r = bits + np.uint64((1 << 44) - 1) + lsb
    r &= ~np.uint64((1 << 45) - 1)
    f32 = r.view(np.float64).astype(np.float32)
    out = (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    tiny = np.abs(x) < 2.0 ** -126
    if tiny.any():
        # bf16 subnormal range: a fixed grid of 2^-133
        v = np.rint(x[tiny] * 2.0 ** 133) * 2.0 ** -133
        out[tiny] = (v.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    return out


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    u = (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16))
    return u.view(np.float32).astype(np.float64)


def _streams(seed: int):
    return [np.random.Generator(np.random.PCG64(s))
            for s in np.random.SeedSequence(seed).spawn(N_STREAMS)]


def make_weight(seed: int, V: int, H: int, std: float = W_STD) -> np.ndarray:
    """W[V,H] ~ N(0, std^2) rounded to bf16 (uint16 bits), drawn in blocks of
    W_BLOCK_ROWS rows from the W stream of ``seed``."""
    g = _streams(seed)[_S_W]
    out = np.empty((V, H), dtype=np.uint16)
    for r0 in range(0, V, W_BLOCK_ROWS):
        r1 = min(V, r0 + W_BLOCK_ROWS)
        out[r0:r1] = f64_to_bf16_bits(g.standard_normal((r1 - r0, H)) * std)
    return out


def rms_normalise(h: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """h / sqrt(mean(h^2) + eps) per row, unit weight, float64.  Input
    preparation for the Qwen-shaped forward workload (the final RMSNorm that
    feeds an LM head), not part of the operator."""
    return h / np.sqrt(np.mean(h * h, axis=1, keepdims=True) + eps)


@dataclasses.dataclass
class Workload:
    name: str
    T: int
    H: int
    V: int
    temperature: float
    hidden: np.ndarray            # uint16 bf16 bits [T,H]
    W: Optional[np.ndarray]       # uint16 bf16 bits [V,H]
    targets: np.ndarray           # int64 [T]
    dlogp: np.ndarray             # float32 [T]
    dentropy: np.ndarray          # float32 [T]
    seq_lens: Optional[np.ndarray] = None
    seed: int = 0

    def hidden_f64(self):
        return bf16_bits_to_f64(self.hidden)

    def W_f64(self):
        return bf16_bits_to_f64(self.W)


def make_rows(seed: int, T: int, H: int, V: int, rms: bool = False):
    """hidden[T,H] ~ N(0,1) (optionally RMS-normalised) as bf16 bits and
    targets[T] uniform in [0,V)."""
    s = _streams(seed)
    h = s[_S_HIDDEN].standard_normal((T, H))
    if rms:
        h = rms_normalise(h)
    hidden = f64_to_bf16_bits(h)
    targets = s[_S_TARGET].integers(0, V, size=T, dtype=np.int64)
    return hidden, targets


def tiny(seed: int = 0) -> Workload:
    """T=64, H=256, V=1024, tau=1, dlogp ~ N(0,1), dentropy = 0.01."""
    T, H, V = 64, 256, 1024
    hidden, targets = make_rows(seed, T, H, V)
    s = _streams(seed)
    dlogp = s[_S_DLOGP].standard_normal(T).astype(np.float32)
    return Workload("tiny", T, H, V, 1.0, hidden, make_weight(seed, V, H), targets,
                    dlogp, np.full(T, 0.01, np.float32), seed=seed)


def small(seed: int = 1) -> Workload:
    """T=512, H=1024, V=32768, tau=0.7, per-row advantage dlogp ~ N(0,1),
    dentropy = 0.001."""
    T, H, V = 512, 1024, 32768
    hidden, targets = make_rows(seed, T, H, V)
    s = _streams(seed)
    dlogp = s[_S_DLOGP].standard_normal(T).astype(np.float32)
    return Workload("small", T, H, V, 0.7, hidden, make_weight(seed, V, H), targets,
                    dlogp, np.full(T, 0.001, np.float32), seed=seed)


QWEN_H, QWEN_V = 4096, 151936


def qwen_fwd(seed: int = 2, T: int = 4096, with_weight: bool = True) -> Workload:
    """Qwen3-8B-shaped LM head forward: T=4096, H=4096, V=151936, hidden
    N(0,1) then RMS-normalised, tau = 1."""
    H, V = QWEN_H, QWEN_V
    hidden, targets = make_rows(seed, T, H, V, rms=True)
    W = make_weight(seed, V, H) if with_weight else None
    z = np.zeros(T, np.float32)
    return Workload("qwen_fwd", T, H, V, 1.0, hidden, W, targets, z, z.copy(), seed=seed)


def target_point(seed: int = 2, T: int = 4096, with_weight: bool = True) -> Workload:
    """Forward + backward at T=4096, H=4096, V=151936, tau = 1: the Qwen-shaped
    rows (hidden N(0,1) then RMS-normalised, targets uniform) with per-row
    dlogp ~ N(0,1) and dentropy = 0.001."""
    w = qwen_fwd(seed, T, with_weight)
    w.name = "target_point"
    w.dlogp = _streams(seed)[_S_DLOGP].standard_normal(T).astype(np.float32)
    w.dentropy = np.full(T, 0.001, np.float32)
    return w


def rl_seq_lens(seed: int, n_seq: int = 8, lo: int = 256, hi: int = 1024) -> np.ndarray:
    """8 response lengths drawn uniformly in [256, 1024] (inclusive)."""
    return _streams(seed)[_S_LENGTHS].integers(lo, hi + 1, size=n_seq, dtype=np.int64)


def rl_step(seed: int = 3, with_weight: bool = True) -> Workload:
    """RL actor step: 8 ragged sequences concatenated into one T, H=4096,
    V=151936, dlogp = one N(0,1) advantage per sequence broadcast over its
    tokens, dentropy = 0.001."""
    H, V = QWEN_H, QWEN_V
    lens = rl_seq_lens(seed)
    T = int(lens.sum())
    hidden, targets = make_rows(seed, T, H, V)
    s = _streams(seed)
    adv = s[_S_DLOGP].standard_normal(len(lens))
    dlogp = np.repeat(adv, lens).astype(np.float32)
    W = make_weight(seed, V, H) if with_weight else None
    return Workload("rl_step", T, H, V, 1.0, hidden, W, targets, dlogp,
                    np.full(T, 0.001, np.float32), seq_lens=lens, seed=seed)


SWEEP_T = (1, 7, 64, 513, 2048, 8192)
N_PROBES = 64


def sweep_probes(seed: int = 4, H: int = QWEN_H, V: int = QWEN_V, n: int = N_PROBES):
    """The fixed probe rows of the batch-invariance sweep: hidden, targets and
    per-row gradient seeds (dlogp ~ N(0,1), dentropy = 0.001)."""
    hidden, targets = make_rows(seed, n, H, V)
    dlogp = _streams(seed)[_S_DLOGP].standard_normal(n).astype(np.float32)
    return hidden, targets, dlogp, np.full(n, 0.001, np.float32)


def sweep_batch(T: int, probes, filler_seed: int, H: int = QWEN_H, V: int = QWEN_V):
    """Embed min(T, n_probes) probe rows at random positions of a batch of T
    rows; the other rows are random fillers drawn from ``filler_seed``.
    Returns (hidden, targets, dlogp, dentropy, probe_idx, positions)."""
    ph, pt, pdl, pde = probes
    n = min(T, ph.shape[0])
    s = _streams(filler_seed)
    hidden, targets = make_rows(filler_seed, T, H, V)
    dlogp = s[_S_DLOGP].standard_normal(T).astype(np.float32)
    dent = np.full(T, 0.001, np.float32)
    pos = s[_S_POS].permutation(T)[:n]
    probe_idx = np.arange(n)
    hidden[pos] = ph[:n]
    targets[pos] = pt[:n]
    dlogp[pos] = pdl[:n]
    dent[pos] = pde[:n]
    return hidden, targets, dlogp, dent, probe_idx, pos


# --------------------------------------------------------------------------
# Diffusion transition step (the RL-Kernel B200 report's transition gate,
# h3-runtime-integration-b200 report.json, transition[].shape): B samples of
# L x D latent elements.
TRANSITION_SHAPES = ((3, 257 * 96), (4, 4096 * 96), (2, 8192 * 32))   # (B, n = L * D)


@dataclasses.dataclass
class TransitionCase:
    B: int
    n: int
    x: np.ndarray    # [B, n] float32 latent
    v: np.ndarray    # [B, n] float32 model output
    eps: np.ndarray  # [B, n] float32 standard normal draw for sampling
    a: np.ndarray    # [B] float32 per-sample coefficient of x
    c: np.ndarray    # [B] float32 per-sample coefficient of v
    s: np.ndarray    # [B] float32 per-sample transition std (> 0)


def transition_case(seed: int, B: int, n: int) -> TransitionCase:
    """Seeded float32 inputs: x, v, eps ~ N(0, 1); a ~ U(0.98, 1.02) (a step
    close to the identity), c ~ U(-0.1, -0.01) (a small step along the model
    output), s ~ U(0.05, 0.5)."""
    ss = np.random.SeedSequence([seed, B, n, 0x7A51])
    r = [np.random.default_rng(k) for k in ss.spawn(6)]
    f32 = np.float32
    return TransitionCase(
        B, n,
        r[0].standard_normal((B, n)).astype(f32),
        r[1].standard_normal((B, n)).astype(f32),
        r[2].standard_normal((B, n)).astype(f32),
        r[3].uniform(0.98, 1.02, B).astype(f32),
        r[4].uniform(-0.1, -0.01, B).astype(f32),
        r[5].uniform(0.05, 0.5, B).astype(f32))
