"""The oracle against the hand-derived worked examples in tests/golden/ (CPU only).

Each fixture states its inputs and every output of the forward and backward
(P, LSE, O, D, dS, dV, dK, dQ) as exact expressions derived by hand from the
definitions, so a dropped term, a wrong sign or a transposed operand anywhere in
the oracle's full-matrix path shows up far above rounding."""
import os

import numpy as np
import pytest

import oracle
from tests import oracle_pins as pins

FIXTURES = pins.golden_fixtures()


def test_fixtures_exist():
    assert len(FIXTURES) >= 2


@pytest.mark.parametrize("path", FIXTURES, ids=os.path.basename)
def test_fixture_is_self_consistent(path):
    # the fixture's own arithmetic, independent of the oracle: rows of P sum to 1,
    # rows of dS sum to 0, O = P v, D = rowsum(dO o O), dV = P^T dO
    fx = pins.load_golden(path)
    np.testing.assert_allclose(fx["p"].sum(axis=1), 1.0, atol=1e-15)
    np.testing.assert_allclose(fx["ds"].sum(axis=1), 0.0, atol=1e-15)
    np.testing.assert_allclose(fx["p"] @ fx["v"], fx["o"], atol=1e-15)
    np.testing.assert_allclose(fx["dO"] * fx["o"], fx["D"], atol=1e-15)
    np.testing.assert_allclose(fx["p"].T @ fx["dO"], fx["dv"], atol=1e-15)


def test_oracle_reproduces_the_worked_examples():
    assert pins.check_worked_examples(oracle.default()) is None
