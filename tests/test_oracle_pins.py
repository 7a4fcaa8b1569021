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
