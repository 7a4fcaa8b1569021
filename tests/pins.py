"""Pins of the fp64 oracle against things other than itself.

Each pin returns (ok, detail).  tests/test_oracle_pins.py asserts that every
pin holds; tests/test_oracle_mutations.py plants known mistakes in the oracle
and asserts that each one breaks at least one pin other than the brute force.

What each pin rests on:
  * brute_force_tiny   -- an independent dense numpy brute force (explicit
                          softmax, Shannon entropy, explicit Jacobian);
  * uniform            -- W = 0 or all rows of W equal: p is uniform, so
                          logp = -ln V, entropy = ln V, lse = z0 + ln V;
  * two_level          -- logits with two distinct values per row have a
                          closed-form lse / logp / entropy (V = 2 is the
                          logistic case); very large gaps give the
                          one-hot-dominant limit entropy -> 0, logp -> 0;
  * invariants         -- sum p = 1, 0 <= entropy <= ln V, logp <= 0,
                          max z <= lse <= max z + ln V;
  * shift              -- adding one vector to every row of W shifts each
                          row's logits by a constant: logp and entropy stay;
  * temperature        -- (tau = 0.5, W) and (tau = 1, 2W) give the same
                          logits exactly; the gradients follow by the chain
                          rule;
  * finite_differences -- central differences of
                          L = sum dlogp*logp + dentropy*entropy;
  * dz_rowsum          -- sum_v dz = 0 (both terms of dz sum to zero);
  * uniform_gradient   -- with W = 0: dx = dlogp (onehot - 1/V) / tau, so dW
                          has a closed form and dHidden = 0.
"""
from __future__ import annotations

import math

import numpy as np

import oracle
from oracle import brute
from invariant_lm_head_gemm_b200 import workloads as wl


def _bits(x):
    return wl.f64_to_bf16_bits(np.asarray(x, np.float64))


def _exact_bits(x):
    """bf16 bits of values that must be exactly representable."""
    b = _bits(x)
    assert np.array_equal(wl.bf16_bits_to_f64(b), np.asarray(x, np.float64)), "not bf16-exact"
    return b


def _rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(1e-300, float(np.max(np.abs(b)))))


def _frob(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(1e-300, float(np.linalg.norm(b))))


def brute_force_tiny():
    errs = {}
    for w in (wl.tiny(0), _rand_case(T=16, H=64, V=200, tau=0.7, wstd=0.3, seed=3)):
        lp, en, ls = oracle.forward(w.hidden, w.W, w.targets, w.temperature)
        blp, ben, bls, _, _ = brute.forward(w.hidden, w.W, w.targets, w.temperature)
        dH, dW = oracle.backward(w.hidden, w.W, w.targets, w.temperature, w.dlogp, w.dentropy)
        bdH, bdW, _ = brute.backward(w.hidden, w.W, w.targets, w.temperature, w.dlogp,
                                     w.dentropy)
        errs[w.name] = dict(logp=_rel(lp, blp), entropy=_rel(en, ben), lse=_rel(ls, bls),
                            dH=_frob(dH, bdH), dW=_frob(dW, bdW))
    return all(e < 1e-10 for d in errs.values() for e in d.values()), errs


def uniform():
    rng = np.random.default_rng(11)
    T, H = 3, 64
    bad = []
    for V in (1, 2, 1024, 4099):
        hidden = _bits(rng.standard_normal((T, H)))
        targets = rng.integers(0, V, size=T)
        W0 = np.zeros((V, H), np.uint16)
        lp, en, ls = oracle.forward(hidden, W0, targets, 0.7)
        lnV = math.log(V)
        if _rel(lp, np.full(T, -lnV)) > 1e-13 and V > 1:
            bad.append(("W=0 logp", V, lp))
        if V == 1 and np.max(np.abs(lp)) > 0:
            bad.append(("V=1 logp", lp))
        if np.max(np.abs(en - lnV)) > 1e-12 or np.max(np.abs(ls - lnV)) > 1e-12:
            bad.append(("W=0 entropy/lse", V, en, ls))
        # all rows of W equal to one vector c: z = (h.c)/tau for every v
        c = rng.standard_normal(H) * 0.05
        cb = _bits(c)
        Weq = np.tile(cb, (V, 1))
        tau = float(np.float32(0.7))
        a = wl.bf16_bits_to_f64(hidden) @ wl.bf16_bits_to_f64(cb) / tau
        lp, en, ls = oracle.forward(hidden, Weq, targets, 0.7)
        if np.max(np.abs(lp + lnV)) > 1e-12 or np.max(np.abs(en - lnV)) > 1e-12:
            bad.append(("equal rows logp/entropy", V, lp, en))
        if np.max(np.abs(ls - (a + lnV))) > 1e-12:
            bad.append(("equal rows lse", V, ls, a + lnV))
    return not bad, bad


def _two_level_case(V, H, hi, lo, k, targets):
    """hidden = all ones, so every row has the same logits: W[k] = hi in every
    column and all other rows of W = lo, giving one logit A = H*hi/tau and
    V-1 logits B = H*lo/tau."""
    T = len(targets)
    hidden = _exact_bits(np.ones((T, H)))
    W = np.full((V, H), lo, np.float64)
    W[k] = hi
    return hidden, _exact_bits(W), np.asarray(targets, np.int64)


def two_level():
    bad = []
    H = 64
    tau = float(np.float32(0.7))
    for V, hi, lo, k in ((2, 0.0625, 0.0, 0), (50, 0.0625, -0.03125, 7), (50, 0.5, 0.0, 49),
                         (1000, 1.0, 0.25, 500)):
        targets = [k, (k + 1) % V, (k + V - 1) % V, k]
        hidden, W, targets = _two_level_case(V, H, hi, lo, k, targets)
        lp, en, ls = oracle.forward(hidden, W, targets, tau)
        A, B = H * hi / tau, H * lo / tau
        g = math.log1p((V - 1) * math.exp(B - A))     # lse - A
        lse_cf = A + g
        p_hi = math.exp(-g)
        q = math.exp(B - A - g)
        ent_cf = -p_hi * math.log(p_hi) - (V - 1) * q * math.log(q)
        for t, tg in enumerate(targets):
            logp_cf = (A if tg == k else B) - lse_cf
            for name, got, want in (("lse", ls[t], lse_cf), ("logp", lp[t], logp_cf),
                                    ("entropy", en[t], ent_cf)):
                if abs(got - want) > 1e-12 * max(1.0, abs(want)):
                    bad.append((V, t, name, got, want))
    # one-hot-dominant limit: a gap of 128/tau nats, every target on the top row
    hidden, W, targets = _two_level_case(64, H, 2.0, 0.0, 5, [5, 5, 5])
    lp, en, ls = oracle.forward(hidden, W, targets, tau)
    if not (np.all(np.abs(lp) < 1e-30) and np.all(en >= 0) and np.all(en < 1e-30)):
        bad.append(("one-hot-dominant", lp, en))
    return not bad, bad


def invariants():
    bad = []
    for w in (wl.tiny(0), _rand_case(T=16, H=128, V=777, tau=0.7, wstd=0.2, seed=8)):
        z = oracle.logits(w.hidden, w.W, w.temperature)
        lp, en, ls = oracle.softmax_stats(z, w.targets)
        lnV = math.log(w.V)
        psum = np.exp(z - ls[:, None]).sum(axis=1)
        zmax = z.max(axis=1)
        checks = {
            "sum_p": np.max(np.abs(psum - 1.0)) < 1e-12,
            "entropy_range": bool(np.all(en >= -1e-12) and np.all(en <= lnV + 1e-12)),
            "logp_nonpos": bool(np.all(lp <= 1e-15)),
            "lse_bounds": bool(np.all(zmax <= ls + 1e-12) and np.all(ls <= zmax + lnV + 1e-12)),
            "forward_matches_stats": _rel(oracle.forward(w.hidden, w.W, w.targets,
                                                         w.temperature)[2], ls) == 0.0,
        }
        if not all(checks.values()):
            bad.append((w.name, checks))
    return not bad, bad


def _rand_case(T, H, V, tau, wstd, seed, dent_std=0.5):
    rng = np.random.default_rng(seed)
    return wl.Workload("rand%d" % seed, T, H, V, tau,
                       _bits(rng.standard_normal((T, H))),
                       _bits(rng.standard_normal((V, H)) * wstd),
                       rng.integers(0, V, size=T).astype(np.int64),
                       rng.standard_normal(T).astype(np.float32),
                       (rng.standard_normal(T) * dent_std).astype(np.float32))


def shift():
    rng = np.random.default_rng(21)
    T, H, V, tau = 8, 96, 300, 0.7
    hidden = _bits(rng.standard_normal((T, H)))
    Wk = rng.integers(-8, 9, size=(V, H)) / 64.0
    ck = rng.integers(-8, 9, size=H) / 64.0
    W = _exact_bits(Wk)
    W2 = _exact_bits(Wk + ck[None, :])
    targets = rng.integers(0, V, size=T)
    lp, en, ls = oracle.forward(hidden, W, targets, tau)
    lp2, en2, ls2 = oracle.forward(hidden, W2, targets, tau)
    shift_t = wl.bf16_bits_to_f64(hidden) @ ck / float(np.float32(tau))
    errs = dict(logp=float(np.max(np.abs(lp - lp2))), entropy=float(np.max(np.abs(en - en2))),
                lse=float(np.max(np.abs(ls2 - ls - shift_t))))
    return all(e < 1e-11 for e in errs.values()), errs


def temperature():
    w = _rand_case(T=8, H=64, V=200, tau=0.5, wstd=0.3, seed=31)
    W2 = _exact_bits(2.0 * wl.bf16_bits_to_f64(w.W))
    a = oracle.forward(w.hidden, w.W, w.targets, 0.5)
    b = oracle.forward(w.hidden, W2, w.targets, 1.0)
    dHa, dWa = oracle.backward(w.hidden, w.W, w.targets, 0.5, w.dlogp, w.dentropy)
    dHb, dWb = oracle.backward(w.hidden, W2, w.targets, 1.0, w.dlogp, w.dentropy)
    errs = dict(fwd=max(_rel(x, y) for x, y in zip(a, b)),
                dH=_frob(dHa, dHb),          # 2 dz . W  ==  dz . 2W
                dW=_frob(dWa, 2.0 * dWb))    # (2 dz)^T h == 2 (dz^T h)
    return all(e < 1e-13 for e in errs.values()), errs


def finite_differences(n_entries=64, eps=1e-5):
    w = _rand_case(T=6, H=64, V=64, tau=0.7, wstd=0.3, seed=41)   # V == H on purpose
    tau = float(np.float32(w.temperature))
    x = oracle.logits(w.hidden, w.W, 1.0)                          # pre-temperature logits
    hd = wl.bf16_bits_to_f64(w.hidden)
    Wd = wl.bf16_bits_to_f64(w.W)
    dl = w.dlogp.astype(np.float64)
    de = w.dentropy.astype(np.float64)

    def L(xx):
        lp, en, _ = oracle.softmax_stats(xx / tau, w.targets)
        return float(np.dot(dl, lp) + np.dot(de, en))

    dx = oracle.dlogits(x / tau, w.targets, tau, dl, de)
    dH = oracle.dhidden(dx, w.W)
    dW = oracle.dw(dx, w.hidden)
    rng = np.random.default_rng(42)
    fd_h, an_h, fd_w, an_w = [], [], [], []
    for _ in range(n_entries):
        t, h = rng.integers(0, w.T), rng.integers(0, w.H)
        xp, xm = x.copy(), x.copy()
        xp[t] += eps * Wd[:, h]
        xm[t] -= eps * Wd[:, h]
        fd_h.append((L(xp) - L(xm)) / (2 * eps))
        an_h.append(dH[t, h])
        v, h = rng.integers(0, w.V), rng.integers(0, w.H)
        xp, xm = x.copy(), x.copy()
        xp[:, v] += eps * hd[:, h]
        xm[:, v] -= eps * hd[:, h]
        fd_w.append((L(xp) - L(xm)) / (2 * eps))
        an_w.append(dW[v, h])
    errs = dict(dHidden=_rel(an_h, fd_h), dW=_rel(an_w, fd_w))
    return all(e < 1e-6 for e in errs.values()), errs


def dz_rowsum():
    w = _rand_case(T=8, H=64, V=500, tau=0.7, wstd=0.3, seed=51)
    z = oracle.logits(w.hidden, w.W, w.temperature)
    dx = oracle.dlogits(z, w.targets, w.temperature, w.dlogp, w.dentropy)
    r = np.abs(dx.sum(axis=1)) / np.abs(dx).sum(axis=1)
    return float(r.max()) < 1e-13, float(r.max())


def uniform_gradient():
    rng = np.random.default_rng(61)
    T, H, V, tau = 8, 64, 37, float(np.float32(0.7))
    hidden = _bits(rng.standard_normal((T, H)))
    targets = rng.integers(0, V, size=T)
    dl = rng.standard_normal(T)
    de = rng.standard_normal(T)
    W0 = np.zeros((V, H), np.uint16)
    dH, dW = oracle.backward(hidden, W0, targets, tau, dl, de)
    onehot = np.zeros((T, V))
    onehot[np.arange(T), targets] = 1.0
    dx_cf = dl[:, None] * (onehot - 1.0 / V) / tau
    dW_cf = dx_cf.T @ wl.bf16_bits_to_f64(hidden)
    errs = dict(dW=_frob(dW, dW_cf), dH=float(np.max(np.abs(dH))))
    return errs["dW"] < 1e-13 and errs["dH"] == 0.0, errs


PINS = {
    "brute_force_tiny": brute_force_tiny,
    "uniform": uniform,
    "two_level": two_level,
    "invariants": invariants,
    "shift": shift,
    "temperature": temperature,
    "finite_differences": finite_differences,
    "dz_rowsum": dz_rowsum,
    "uniform_gradient": uniform_gradient,
}


def run_pin(name):
    try:
        return PINS[name]()
    except (AssertionError, ValueError, FloatingPointError, ZeroDivisionError) as e:
        return False, "raised %r" % (e,)
