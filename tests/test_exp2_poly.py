"""The FMA-pipe exp2 of the prefill softmax: its constants are the minimax fit they claim
to be, and the reduction + polynomial + exponent-add steps give 2^x to 3e-6 relative."""
import numpy as np

from exact_io_aware_59_b200 import exp2_poly


def test_header_constants_are_the_minimax_fit():
    c, err = exp2_poly.minimax_coefficients()
    assert err < 2.7e-6
    np.testing.assert_allclose(exp2_poly.header_coefficients(), c, rtol=0, atol=2e-7)


def test_emulated_exp2_accuracy_over_the_softmax_range():
    c = exp2_poly.header_coefficients()
    x = np.concatenate([np.linspace(-125.0, 16.0, 400001, dtype=np.float32),
                        np.array([0.0, -0.5, 0.5, 1.0, -1.0, 8.0, -125.0], dtype=np.float32)])
    got = exp2_poly.exp2_emulated(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got / ref - 1)) < 3e-6


def test_emulated_exp2_clamps_far_below():
    c = exp2_poly.header_coefficients()
    x = np.array([-125.5, -126.0, -127.0, -200.0, -1e30, -np.inf], dtype=np.float32)
    got = exp2_poly.exp2_emulated(x, c)
    # clamped to 2^-125 (a normal number, negligible against a row sum >= 1)
    assert np.all(got > 0) and np.all(got < 2.4e-38)
