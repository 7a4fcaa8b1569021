"""The fp64 oracle against its pins (closed forms, invariants, brute force,
finite differences); no GPU needed."""
import pytest

from tests import pins


@pytest.mark.parametrize("name", list(pins.PINS))
def test_pin(name):
    ok, detail = pins.run_pin(name)
    assert ok, detail


def test_oracle_rejects_out_of_range_targets():
    """The oracle refuses a target outside [0, V) (the GPU path instead returns
    NaN logp for that row and sets its error flag; tested on the GPU)."""
    import numpy as np
    import pytest as _pytest

    import oracle
    from invariant_lm_head_gemm_b200 import workloads as wl
    w = wl.tiny(0)
    for bad in (-1, w.V):
        t = np.array(w.targets, copy=True)
        t[3] = bad
        with _pytest.raises(ValueError):
            oracle.forward(w.hidden, w.W, t, w.temperature)
        with _pytest.raises(ValueError):
            oracle.backward(w.hidden, w.W, t, w.temperature, w.dlogp, w.dentropy)


@__import__("pytest").mark.parametrize("seed", range(12))
def test_oracle_matches_brute_force_on_random_small_shapes(seed):
    """A randomized sweep of small shapes, temperatures and weight scales
    (ragged T, V not a multiple of anything, tiny and large logits) against
    the independent dense brute force: the oracle's two-pass softmax, its
    entropy form and its gradient must agree with the textbook routes."""
    import numpy as np

    import oracle
    from oracle import brute
    from tests import pins
    rng = np.random.default_rng(1000 + seed)
    T = int(rng.integers(1, 20))
    H = int(rng.choice([64, 128, 192]))
    V = int(rng.integers(2, 300))
    tau = float(rng.choice([0.25, 0.7, 1.0, 1.9]))
    wstd = float(rng.choice([0.01, 0.1, 0.5]))
    w = pins._rand_case(T=T, H=H, V=V, tau=tau, wstd=wstd, seed=seed)
    lp, en, ls = oracle.forward(w.hidden, w.W, w.targets, w.temperature)
    blp, ben, bls, _, _ = brute.forward(w.hidden, w.W, w.targets, w.temperature)
    dH, dW = oracle.backward(w.hidden, w.W, w.targets, w.temperature, w.dlogp, w.dentropy)
    bdH, bdW, _ = brute.backward(w.hidden, w.W, w.targets, w.temperature, w.dlogp, w.dentropy)
    for got, ref in ((lp, blp), (en, ben), (ls, bls)):
        np.testing.assert_allclose(got, ref, rtol=1e-9, atol=1e-11)
    for got, ref in ((dH, bdH), (dW, bdW)):
        assert np.linalg.norm(got - ref) <= 1e-9 * max(np.linalg.norm(ref), 1e-300)
