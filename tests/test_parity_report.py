"""CPU checks of the parity helpers: the bounds they apply and the record of
every comparison (the elementwise allclose reading and its worst element)."""

import numpy as np
import pytest

import parity


def test_plain_bound_records_elementwise_reading():
    want = np.array([[0.0, 1.0], [10.0, -2.0]])
    got = want + np.array([[0.019, 0.0], [0.0, -0.001]])
    n0 = len(parity.RECORDS)
    parity.assert_close(got, want, "t")
    r = parity.RECORDS[n0]
    assert r["what"] == "t" and r["pass"]
    assert abs(r["max_abs"] - 0.019) < 1e-12
    # |err| <= 2e-2 + 1e-2 |want| everywhere
    assert r["allclose"] and r["frac_outside"] == 0.0
    assert r["worst"]["index"] == [0, 0]


def test_elementwise_worst_element_is_the_one_furthest_past_its_allowance():
    want = np.array([0.0, 5.0, 100.0])
    # allowances 0.02, 0.07, 1.02; excesses 0.01, 0.13, -0.52
    got = want + np.array([0.03, 0.2, 0.5])
    e = parity.elementwise(got, want)
    assert not e["allclose"]
    assert e["worst"]["index"] == [1]
    assert abs(e["frac_outside"] - 2 / 3) < 1e-12


def test_plain_bound_fails_on_large_absolute_error():
    want = np.ones(16)
    with pytest.raises(AssertionError):
        parity.assert_close(want + 0.03, want, "over")
    assert parity.RECORDS[-1]["pass"] is False


def test_scaled_bound_scales_only_above_unit_size():
    want = np.full(100, 10.0)
    got = want.copy()
    got[3] += 0.15  # over 2e-2, under 2e-2 * 10; relL2 = 1.5e-3
    parity.assert_close_scaled(got, want, "dW")
    r = parity.RECORDS[-1]
    assert r["pass"] and "*10" in r["bound"] and abs(r["max_abs_over_max_ref"] - 0.015) < 1e-12
    small = np.full(100, 0.5)
    with pytest.raises(AssertionError):  # scale is max(1, max|ref|) = 1 here
        parity.assert_close_scaled(small + 0.03, small, "small")
