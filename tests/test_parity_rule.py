"""The comparison rule of the GPU parity tests, checked on the CPU with
made-up arrays: every element within 2e-2 of the oracle and the mean within
2e-3, except that an entry whose oracle value is itself farther than 2e-2
from every bf16 number (|ref| >= 8) may miss by that distance more, and such
entries are reported."""
import numpy as np
import pytest

import parity


def test_small_entries_held_to_the_bar():
    ref = np.array([3.0, -5.5, 0.25, 7.9])
    parity.assert_close("ok", ref + 0.0199, ref, tol_mean=None)
    with pytest.raises(AssertionError):
        parity.assert_close("over", ref + np.array([0, 0, 0.0201, 0]), ref, tol_mean=None)


def test_large_entries_get_their_rounding_distance_and_are_reported():
    parity.LOOSENED.clear()
    ref = np.array([1.0, 8.0 + 0.0625 * 0.5, -12.03])      # the last two have floors > 2e-2
    floor = parity.rounding_distance(ref)
    assert floor[0] == 0.0 and floor[1] > 2e-2 and floor[2] > 2e-2
    got = ref + np.array([0.0, 2e-2 + 0.9 * floor[1], -(2e-2 + 0.9 * floor[2])])
    parity.assert_close("big", got, ref, tol_mean=None)
    assert parity.LOOSENED and parity.LOOSENED[-1][0] == "big" and parity.LOOSENED[-1][1] == 2
    with pytest.raises(AssertionError):
        parity.assert_close("big2", ref + np.array([0.0, 2e-2 + 1.1 * floor[1], 0.0]), ref,
                            tol_mean=None)


def test_mean_bound_and_non_bf16_outputs():
    ref = np.zeros(1000)
    with pytest.raises(AssertionError):
        parity.assert_close("mean", ref + 2.5e-3, ref)            # every entry under 2e-2
    lse = np.array([100.0, -50.0])
    parity.assert_close("lse", lse + 9e-4, lse, tol_max=1e-3, tol_mean=None, bf16_out=False)
    with pytest.raises(AssertionError):
        parity.assert_close("lse", lse + 1.1e-3, lse, tol_max=1e-3, tol_mean=None,
                            bf16_out=False)


def test_non_finite_output_fails():
    with pytest.raises(AssertionError):
        parity.assert_close("nan", np.array([np.nan, 0.0]), np.zeros(2))
