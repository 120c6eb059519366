"""The oracle against its pins (CPU only)."""
import pytest

import oracle
import pins


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda f: f.__name__)
def test_pin(check):
    check(oracle.get())


def test_threads_do_not_change_results():
    import numpy as np
    x = pins._randn_bf16((97, 64), 40)
    r = pins._randn_bf16((97, 64), 41)
    o = oracle.get()
    y1, h1 = o.add_rms_norm(x, r, None, 1e-5, threads=1)
    y4, h4 = o.add_rms_norm(x, r, None, 1e-5, threads=4)
    assert o.last_threads == 4
    assert (y1 == y4).all() and (h1 == h4).all()
    assert np.isfinite(y1).all()
