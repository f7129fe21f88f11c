"""The oracle against the hand-derived worked examples in tests/golden/ (CPU only).

Each fixture states its inputs and every output of the forward and backward
(P, LSE, O, D, dS, dV, dK, dQ) as exact expressions derived by hand from the
definitions, so a dropped term, a wrong sign or a transposed operand anywhere in
the oracle shows up as a mismatch far above rounding."""
import glob
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
FIXTURES = sorted(glob.glob(os.path.join(GOLDEN, "worked_*.txt")))


def _eval(expr: str) -> float:
    return float(eval(expr, {"__builtins__": {}}, {"log": math.log}))


def _split(rhs: str):
    # split on commas outside parentheses
    out, depth, cur = [], 0, ""
    for ch in rhs:
        if ch == "," and depth == 0:
            out.append(cur)
            cur = ""
            continue
        depth += ch == "("
        depth -= ch == ")"
        cur += ch
    out.append(cur)
    return [_eval(e.strip()) for e in out if e.strip()]


def load_fixture(path):
    vec, mat = {}, {}
    for line in open(path):
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        lhs, rhs = (s.strip() for s in line.split("=", 1))
        vals = _split(rhs)
        if "[" in lhs:
            name, idx = lhs[:-1].split("[")
            mat.setdefault(name, {})[int(idx)] = vals
        else:
            vec[lhs] = vals
    for name, rows in mat.items():
        vec[name] = [rows[i] for i in range(len(rows))]
    return {k: np.array(v, dtype=np.float64) for k, v in vec.items()}


def test_fixtures_exist():
    assert len(FIXTURES) >= 2


@pytest.mark.parametrize("path", FIXTURES, ids=os.path.basename)
def test_oracle_reproduces_worked_example(path):
    fx = load_fixture(path)
    orc = oracle.default()
    scale, causal = float(fx["scale"][0]), int(fx["causal"][0])
    q, k, v, dO = (fx[n].reshape(-1, 1) for n in ("q", "k", "v", "dO"))
    o, lse, p = orc.fwd_head(q, k, v, scale, causal, want_p=True)
    dq, dk, dv, ds, dvec = orc.bwd_head(q, k, v, dO, scale, causal, want_ds=True)
    got = {"p": p, "lse": lse, "o": o[:, 0], "D": dvec, "ds": ds, "dv": dv[:, 0],
           "dk": dk[:, 0], "dq": dq[:, 0]}
    for name, value in got.items():
        np.testing.assert_allclose(value, fx[name], rtol=0, atol=1e-13, err_msg=name)


def test_worked_example_is_self_consistent():
    # the fixtures' own arithmetic, independent of the oracle: rows of P sum to 1,
    # rows of dS sum to 0, O = P v, D = rowsum(dO o O)
    for path in FIXTURES:
        fx = load_fixture(path)
        np.testing.assert_allclose(fx["p"].sum(axis=1), 1.0, atol=1e-15)
        np.testing.assert_allclose(fx["ds"].sum(axis=1), 0.0, atol=1e-15)
        np.testing.assert_allclose(fx["p"] @ fx["v"], fx["o"], atol=1e-15)
        np.testing.assert_allclose(fx["dO"] * fx["o"], fx["D"], atol=1e-15)
