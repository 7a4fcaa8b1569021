"""fp64 CPU oracle for the diffusion transition step and its log-probability
-- TEST INFRASTRUCTURE ONLY (only tests/, __graft_entry__.smoke() and the
CPU-baseline leg of bench.py may use it; the CUDA library never does).

What it follows.  The B200 runtime-integration report of RL-Kernel
(h3-runtime-integration-b200 report.json, the "transition" gate) checks a
diffusion transition operator on shapes B3 x 257x96, B4 x 4096x96 and
B2 x 8192x32: the sampled prev_sample and the transition mean are bitwise
equal between paths, the per-sample log-probability is within
logp_max_rel_diff_vs_torch_mean (5.8e-6 .. 1.5e-4) of a torch computation
that averages over the element dimensions, and it is batch invariant, with
scoring reproducing the sampling log-probability.  The report gives no
formula.  The reading taken here (the plainest one those fields support): a
Gaussian transition with an affine mean,

    mean = a_b * x + c_b * v                       (x: latent, v: model output)
    prev = mean + s_b * eps                        (sampling; eps ~ N(0, 1) given)
    logp_b = (1 / n) * sum_i [ -(prev_i - mean_i)^2 / (2 s_b^2) - ln s_b - ln(2 pi) / 2 ]

with per-sample scalars a_b, c_b, s_b > 0 (whatever sampler schedule produced
them) and the mean taken over the n = L * D elements of each sample.

Arrays are float arrays [B, n] (any float dtype, widened to float64 exactly);
coefficients are [B].

Pinned by tests/test_transition_oracle.py: scipy.stats.norm.logpdf averaged
per sample, the sampling identity logp = -mean(eps^2)/2 - ln s - ln(2 pi)/2,
the zero-residual value, the change-of-variables shift under scaling, a
hand-worked two-element case (tests/golden/transition_hand.json) and
per-sample independence.
"""
from __future__ import annotations

import math

import numpy as np

# One known mistake at a time can be planted for the mutation tests.
_MUTATION = 0
MUTATIONS = {1: "no_log_s", 2: "residual_sign", 3: "s_not_squared", 4: "c_times_x",
             5: "sum_not_mean", 6: "a_c_swapped", 7: "sample_without_s"}


class mutation:
    """Context manager that plants mutation `code` (see MUTATIONS)."""

    def __init__(self, code: int):
        self.code = code

    def __enter__(self):
        global _MUTATION
        _MUTATION = self.code
        return self

    def __exit__(self, *exc):
        global _MUTATION
        _MUTATION = 0
        return False


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def transition_mean(x, v, a, c):
    """mean[b, i] = a_b x[b, i] + c_b v[b, i]."""
    x, v = _f64(x), _f64(v)
    a, c = _f64(a)[:, None], _f64(c)[:, None]
    if _MUTATION == 4:
        return a * x + c * x
    if _MUTATION == 6:
        return c * x + a * v
    return a * x + c * v


def gaussian_logp(prev, mean, s):
    """Per-sample mean over elements of the N(mean, s_b^2) log-density of prev."""
    prev, mean = _f64(prev), _f64(mean)
    s = _f64(s)[:, None]
    r = prev - mean
    var2 = 2.0 * s if _MUTATION == 3 else 2.0 * s * s
    quad = (r * r) / var2
    if _MUTATION == 2:
        quad = -quad
    log_s = 0.0 if _MUTATION == 1 else np.log(s)
    elem = -quad - log_s - 0.5 * math.log(2.0 * math.pi)
    if _MUTATION == 5:
        return elem.sum(axis=1)
    return elem.mean(axis=1)


def transition_sample(x, v, eps, a, c, s):
    """(mean, prev, logp) of one sampling step with noise eps."""
    mean = transition_mean(x, v, a, c)
    scale = np.ones_like(_f64(s)) if _MUTATION == 7 else _f64(s)
    prev = mean + scale[:, None] * _f64(eps)
    return mean, prev, gaussian_logp(prev, mean, s)


def transition_logp(x, v, prev, a, c, s):
    """(mean, logp) of scoring a recorded prev_sample."""
    mean = transition_mean(x, v, a, c)
    return mean, gaussian_logp(prev, mean, s)
