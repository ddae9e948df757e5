"""The fp64 oracle against its pins (finite differences, torch autograd, scipy,
closed forms and invariants).  See oracle_pins.py for what each one fixes."""
import pytest

import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_rows_mode_matches_full(orc):
    """rows(r0, n) reproduces the full call on those rows, and under the causal
    mask its dY contribution is the exact dY_s for columns >= r0."""
    import numpy as np
    rng = np.random.default_rng(3)
    n, d = 70, 8
    Xt, Yt, Xs, Ys = (rng.standard_normal((n, d)) for _ in range(4))
    full = orc.relation(Xt[None], Yt[None], Xs[None], Ys[None], 0.3, True)
    r0 = 41
    part = orc.rows(Xt, Yt, Xs, Ys, 0.3, True, r0, n, want_dY=True)
    np.testing.assert_allclose(part["lse_t"], full["lse_t"][0, r0:], rtol=0, atol=1e-13)
    np.testing.assert_allclose(part["lse_s"], full["lse_s"][0, r0:], rtol=0, atol=1e-13)
    np.testing.assert_allclose(part["row_kl"], full["row_kl"][0, r0:], rtol=0, atol=1e-13)
    np.testing.assert_allclose(part["dXs"], full["dXs"][0, r0:], rtol=0, atol=1e-15)
    np.testing.assert_allclose(part["dYs"][r0:], full["dYs"][0, r0:], rtol=0, atol=1e-15)


def test_threads_reported(orc):
    assert orc.num_threads() >= 1
