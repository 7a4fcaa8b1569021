"""Pins of the fp64 transition oracle (oracle/transition.py) against what
does not come from its own code: scipy's normal log-density, closed forms,
special cases, a hand-worked example and change of variables.  Each planted
mistake must trip at least one of them.  Shapes follow the RL-Kernel B200
report's transition gate (h3-runtime-integration-b200 report.json,
transition[].shape: B3 x 257x96, B4 x 4096x96, B2 x 8192x32)."""
import json
import math
import os

import numpy as np
import pytest
from scipy import stats

from oracle import transition as tr
from invariant_lm_head_gemm_b200 import workloads as wl

HALF_LOG_2PI = 0.5 * math.log(2.0 * math.pi)
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "transition_hand.json")


def _case(B=3, n=257 * 96, seed=0):
    w = wl.transition_case(seed, B, n)
    w.s = w.s.astype(np.float64)   # exact widening, so that the pins' own logs are fp64
    return w


def pin_scipy():
    w = _case()
    mean, prev, logp = tr.transition_sample(w.x, w.v, w.eps, w.a, w.c, w.s)
    ref = stats.norm.logpdf(prev, loc=mean, scale=np.asarray(w.s)[:, None]).mean(axis=1)
    return np.allclose(logp, ref, rtol=1e-12, atol=0.0)


def pin_sampling_identity():
    w = _case(B=2, n=8192 * 32, seed=1)
    mean, prev, logp = tr.transition_sample(w.x, w.v, w.eps, w.a, w.c, w.s)
    eps = np.asarray(w.eps, np.float64)
    closed = -0.5 * (eps * eps).mean(axis=1) - np.log(w.s) - HALF_LOG_2PI
    resid_ok = np.allclose(prev - mean, np.asarray(w.s)[:, None] * eps, rtol=1e-12, atol=1e-15)
    return resid_ok and np.allclose(logp, closed, rtol=1e-12, atol=0.0)


def pin_zero_residual():
    w = _case(B=4, n=96, seed=2)
    mean = tr.transition_mean(w.x, w.v, w.a, w.c)
    _, logp = tr.transition_logp(w.x, w.v, mean, w.a, w.c, w.s)
    return np.allclose(logp, -np.log(w.s) - HALF_LOG_2PI, rtol=1e-14, atol=0.0)


def pin_mean_special_cases():
    w = _case(B=3, n=64, seed=3)
    zeros = np.zeros_like(np.asarray(w.x, np.float64))
    only_x = tr.transition_mean(w.x, zeros, w.a, w.c)
    only_v = tr.transition_mean(zeros, w.v, w.a, w.c)
    a, c = np.asarray(w.a)[:, None], np.asarray(w.c)[:, None]
    return (np.array_equal(only_x, a * np.asarray(w.x, np.float64)) and
            np.array_equal(only_v, c * np.asarray(w.v, np.float64)))


def pin_change_of_variables():
    # scaling x, v, eps and s by k scales prev - mean by k: the density of a
    # scaled variable gains -ln k per element, so the per-element mean shifts
    # by exactly -ln k
    w = _case(B=2, n=1000, seed=4)
    k = 3.0
    _, _, l1 = tr.transition_sample(w.x, w.v, w.eps, w.a, w.c, w.s)
    _, _, l2 = tr.transition_sample(k * np.asarray(w.x, np.float64),
                                    k * np.asarray(w.v, np.float64),
                                    np.asarray(w.eps, np.float64), w.a, w.c,
                                    k * np.asarray(w.s, np.float64))
    return np.allclose(l2, l1 - math.log(k), rtol=0.0, atol=1e-12)


def pin_hand_worked():
    g = json.load(open(GOLDEN))
    mean, logp = tr.transition_logp(g["x"], g["v"], g["prev"], g["a"], g["c"], g["s"])
    return (np.allclose(mean, g["mean"], rtol=0, atol=0) and
            np.allclose(logp, g["logp"], rtol=1e-15, atol=0) and
            math.isclose(g["logp"][0], -1.25 + math.log(2.0) - HALF_LOG_2PI, rel_tol=1e-15))


def pin_per_sample_independence():
    w = _case(B=4, n=4096, seed=5)
    _, _, full = tr.transition_sample(w.x, w.v, w.eps, w.a, w.c, w.s)
    x, v, e = (np.asarray(t) for t in (w.x, w.v, w.eps))
    a, c, s = (np.asarray(t) for t in (w.a, w.c, w.s))
    alone = [tr.transition_sample(x[b:b + 1], v[b:b + 1], e[b:b + 1], a[b:b + 1], c[b:b + 1],
                                  s[b:b + 1])[2][0] for b in (3, 0, 2, 1)]
    return np.array_equal(np.array(alone), full[[3, 0, 2, 1]])


PINS = {f.__name__[4:]: f for f in (pin_scipy, pin_sampling_identity, pin_zero_residual,
                                     pin_mean_special_cases, pin_change_of_variables,
                                     pin_hand_worked, pin_per_sample_independence)}


@pytest.mark.parametrize("name", sorted(PINS))
def test_pin_holds(name):
    assert PINS[name]()


@pytest.mark.parametrize("code", sorted(tr.MUTATIONS))
def test_mutation_is_caught(code):
    with tr.mutation(code):
        failed = [n for n, f in PINS.items() if not f()]
    assert failed, "mutation %s went unnoticed" % tr.MUTATIONS[code]
    assert "hand_worked" in failed or code == 7    # sampling-only mistake: no eps in that case
    assert [n for n in failed if n != "hand_worked"], tr.MUTATIONS[code]


def test_pins_hold_after_mutations():
    assert all(f() for f in PINS.values())
