"""Plant one plausible mistake at a time in a copy of the oracle's C source and
check that the pins catch every one (CPU only).  The shipped oracle is untouched:
each mutant is compiled into a temporary directory."""
import os

import pytest

import oracle
from tests import oracle_pins as pins

MUTATIONS = {
    "scale dropped from S": ("srow[j] = masked(causal, i, j) ? -INFINITY : scale * srow[j];",
                             "srow[j] = masked(causal, i, j) ? -INFINITY : srow[j];"),
    "mask off by one": ("return causal && j > i;", "return causal && j >= i + 1 && j > i + 1;"),
    "D with the wrong sign": ("dS[x] = P[x] * (S[x] - Dv[i]);", "dS[x] = P[x] * (S[x] + Dv[i]);"),
    "dV not transposed": ("matmul_ttT_td(T, d, P, dO, dv);", "matmul_tt_td(T, d, P, dO, dv);"),
    "scale dropped from dQ": ("for (size_t x = 0; x < td; ++x) dq[x] *= scale;", ""),
    "dK from K instead of Q": ("matmul_ttT_td(T, d, dS, q, dk);",
                               "matmul_ttT_td(T, d, dS, kk, dk);"),
    "row max dropped from LSE": ("        const double l = m + log(sum);\n        lse[i] = l;",
                                 "        const double l = log(sum);\n        lse[i] = l;"),
    "wrong row of V in P V": ("const double* brow = B + (size_t)j * d;\n            for (int c = 0; c < d; ++c) crow[c] += a * brow[c];",
                              "const double* brow = B + (size_t)i * d;\n            for (int c = 0; c < d; ++c) crow[c] += a * brow[c];"),
    "dP from O instead of V": ("s += dO[(size_t)i * d + c] * v[(size_t)j * d + c];\n            S[(size_t)i * T + j] = s;",
                               "s += dO[(size_t)i * d + c] * O[(size_t)j * d + c];\n            S[(size_t)i * T + j] = s;"),
    "row sampler: dK without scale": ("            if (dkr)\n                for (int c = 0; c < d; ++c) dkr[c] *= scale;", ""),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, tmp_path):
    src = open(oracle.SOURCE).read()
    old, new = MUTATIONS[name]
    assert src.count(old) == 1, f"mutation anchor not found exactly once: {name}"
    path = os.path.join(tmp_path, "mutant.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = oracle.build(path, os.path.join(tmp_path, "libmutant.so"))
    failures = pins.all_checks(oracle.Oracle(lib))
    assert failures, f"no pin caught: {name}"


# Every planted mistake in the full-matrix path (all but the row sampler's) is also
# caught by the hand-derived worked examples alone.
@pytest.mark.parametrize("name", sorted(n for n in MUTATIONS if not n.startswith("row sampler")))
def test_worked_examples_alone_catch_mutation(name, tmp_path):
    src = open(oracle.SOURCE).read()
    old, new = MUTATIONS[name]
    path = os.path.join(tmp_path, "mutant.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = oracle.build(path, os.path.join(tmp_path, "libmutant.so"))
    try:
        msg = pins.check_worked_examples(oracle.Oracle(lib))
    except Exception as e:  # a crash in a mutated oracle counts as caught
        msg = repr(e)
    assert msg, f"the worked examples did not catch: {name}"
