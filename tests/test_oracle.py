"""The fp64 oracle against its pins (CPU only)."""
import numpy as np
import pytest

import oracle
from oracle_pins import PIN_TOL, rand_case


@pytest.mark.parametrize("pin", list(PIN_TOL), ids=lambda f: f.__name__)
def test_pin(pin):
    err = pin()
    assert err <= PIN_TOL[pin], f"{pin.__name__}: deviation {err:.3e}"


def test_decode_step_is_one_token_of_fwd():
    rng = np.random.default_rng(11)
    q, k, v, g, beta, h0 = rand_case(rng, T=1, B=3, H=2, dk=4, dv=6)
    out, s = oracle.kda_decode_step(q[:, 0], k[:, 0], v[:, 0], g[:, 0], beta[:, 0], 0.3, h0)
    out2, s2 = oracle.kda_fwd(q, k, v, g, beta, 0.3, h0)
    assert np.array_equal(out, out2[:, 0]) and np.array_equal(s, s2)


def test_threads_do_not_change_result():
    rng = np.random.default_rng(12)
    q, k, v, g, beta, h0 = rand_case(rng, B=3, H=5, T=33)
    a = oracle.kda_fwd(q, k, v, g, beta, 0.5, h0, threads=1)
    b = oracle.kda_fwd(q, k, v, g, beta, 0.5, h0, threads=4)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_zero_length_sequence_returns_h0():
    rng = np.random.default_rng(13)
    q, k, v, g, beta, h0 = rand_case(rng, T=0)
    out, hT = oracle.kda_fwd(q, k, v, g, beta, 0.5, h0)
    assert out.shape[1] == 0 and np.array_equal(hT, h0)


def test_shape_errors():
    rng = np.random.default_rng(14)
    q, k, v, g, beta, h0 = rand_case(rng)
    with pytest.raises(ValueError):
        oracle.kda_fwd(q, k[:, :-1], v, g, beta, 1.0, h0)
    with pytest.raises(ValueError):
        oracle.kda_fwd(q, k, v, g, beta[..., :-1], 1.0, h0)
    with pytest.raises(ValueError):
        oracle.kda_fwd(q, k, v, g, beta, 1.0, h0[..., :-1])
