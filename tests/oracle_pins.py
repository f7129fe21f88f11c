"""Independent checks that pin the fp64 oracle to the mathematics.

Each check returns None when it passes and a short message when it fails, so the
same suite can be run against the shipped oracle (tests/test_oracle.py) and
against copies with a planted mistake (tests/test_oracle_mutations.py).

None of these re-types the oracle's own formulas:
  * brute force uses the textbook softmax-attention formula exp(s)/sum exp(s)
    with no max subtraction and no log-sum-exp, summed with math.fsum;
  * gradients are central finite differences of L = sum(dO o O), which uses
    only the oracle's forward;
  * closed forms: Q = 0 gives uniform weights over the allowed keys, T = 1 gives
    O = v0, LSE = scale q0.k0 and zero dQ, dK with dV = dO;
  * invariants: softmax rows sum to 1, row i ignores keys > i under the causal
    mask, each row of dS sums to 0, and dO = 0 gives zero gradients;
  * worked examples (tests/golden/): every forward and backward output of a small
    case stated as an exact expression derived by hand.
"""
from __future__ import annotations

import glob
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def brute_fwd(q, k, v, scale, causal):
    T, d = q.shape
    O = np.zeros((T, d))
    L = np.zeros(T)
    for i in range(T):
        js = [j for j in range(T) if not (causal and j > i)]
        w = [math.exp(scale * math.fsum(q[i, c] * k[j, c] for c in range(d))) for j in js]
        Z = math.fsum(w)
        L[i] = math.log(Z)
        for c in range(d):
            O[i, c] = math.fsum(w[n] * v[j, c] for n, j in enumerate(js)) / Z
    return O, L


def fd_grads(orc, q, k, v, dO, scale, causal, h=1e-5):
    """Central differences of L = sum(dO * O(q, k, v)) with respect to q, k and v."""
    def loss(qq, kk, vv):
        o, _ = orc.fwd_head(qq, kk, vv, scale, causal)
        return float(np.sum(dO * o))

    grads = []
    for which in range(3):
        base = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(base[which])
        for idx in np.ndindex(*g.shape):
            plus = [x.copy() for x in base]
            minus = [x.copy() for x in base]
            plus[which][idx] += h
            minus[which][idx] -= h
            g[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
        grads.append(g)
    return grads


def _rel(a, b):
    den = max(np.linalg.norm(b), 1e-300)
    return float(np.linalg.norm(a - b) / den)


def tiny_case(seed, T, d, sigma=1.0):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((T, d)) * sigma for _ in range(4)]


def check_brute_force(orc, T=7, d=4, causal=1, scale=0.37, seed=1):
    q, k, v, _ = tiny_case(seed, T, d)
    o, lse = orc.fwd_head(q, k, v, scale, causal)
    ob, lb = brute_fwd(q, k, v, scale, causal)
    if np.max(np.abs(o - ob)) > 1e-12 or np.max(np.abs(lse - lb)) > 1e-12:
        return (f"brute force T={T} d={d} causal={causal}: |dO|={np.max(np.abs(o - ob)):.3g} "
                f"|dLSE|={np.max(np.abs(lse - lb)):.3g}")
    return None


def check_finite_differences(orc, T=6, d=4, causal=1, scale=0.61, seed=2):
    q, k, v, dO = tiny_case(seed, T, d)
    dq, dk, dv = orc.bwd_head(q, k, v, dO, scale, causal)
    fq, fk, fv = fd_grads(orc, q, k, v, dO, scale, causal)
    errs = {n: _rel(a, b) for n, a, b in (("dQ", dq, fq), ("dK", dk, fk), ("dV", dv, fv))}
    bad = {n: e for n, e in errs.items() if not e <= 1e-6}
    if bad:
        return f"finite differences T={T} d={d} causal={causal}: rel err {bad}"
    return None


def check_zero_q_closed_form(orc, T=9, d=3, causal=1, scale=0.5, seed=3):
    _, k, v, _ = tiny_case(seed, T, d)
    q = np.zeros((T, d))
    o, lse = orc.fwd_head(q, k, v, scale, causal)
    for i in range(T):
        n = i + 1 if causal else T
        if abs(lse[i] - math.log(n)) > 1e-13:
            return f"Q=0: LSE[{i}]={lse[i]} != ln({n})"
        want = v[:n].mean(axis=0)
        if np.max(np.abs(o[i] - want)) > 1e-13:
            return f"Q=0: O[{i}] is not the mean of v[0..{n - 1}]"
    return None


def check_t1_closed_form(orc, d=5, scale=0.7, seed=4):
    q, k, v, dO = tiny_case(seed, 1, d)
    o, lse = orc.fwd_head(q, k, v, scale, 1)
    dq, dk, dv = orc.bwd_head(q, k, v, dO, scale, 1)
    if np.max(np.abs(o - v)) > 1e-15:
        return "T=1: O != v0"
    if abs(lse[0] - scale * math.fsum(q[0] * k[0])) > 1e-13:
        return "T=1: LSE != scale q0.k0"
    if np.max(np.abs(dq)) > 1e-15 or np.max(np.abs(dk)) > 1e-15:
        return "T=1: dQ or dK not zero"
    if np.max(np.abs(dv - dO)) > 1e-15:
        return "T=1: dV != dO"
    return None


def check_softmax_rows(orc, T=8, d=4, causal=1, scale=0.9, seed=5):
    q, k, v, _ = tiny_case(seed, T, d)
    _, lse, p = orc.fwd_head(q, k, v, scale, causal, want_p=True)
    if np.max(np.abs(p.sum(axis=1) - 1.0)) > 1e-12:
        return "softmax rows do not sum to 1"
    if causal and np.any(np.triu(p, 1) != 0.0):
        return "P is not exactly 0 above the diagonal"
    s = scale * (q @ k.T)
    if causal:
        s = np.where(np.triu(np.ones((T, T), bool), 1), -np.inf, s)
    if np.any(lse < s.max(axis=1) - 1e-12):
        return "LSE < row max"
    return None


def check_causal_independence(orc, T=8, d=4, scale=0.8, seed=6, i0=3):
    q, k, v, dO = tiny_case(seed, T, d)
    o1, l1 = orc.fwd_head(q, k, v, scale, 1)
    k2, v2 = k.copy(), v.copy()
    rng = np.random.default_rng(seed + 100)
    k2[i0 + 1:] += rng.standard_normal(k2[i0 + 1:].shape) * 3
    v2[i0 + 1:] += rng.standard_normal(v2[i0 + 1:].shape) * 3
    o2, l2 = orc.fwd_head(q, k2, v2, scale, 1)
    if not (np.array_equal(o1[:i0 + 1], o2[:i0 + 1]) and np.array_equal(l1[:i0 + 1], l2[:i0 + 1])):
        return "rows <= i0 changed when keys > i0 were perturbed"
    if np.array_equal(o1[i0 + 1:], o2[i0 + 1:]):
        return "rows > i0 did not change when their keys were perturbed"
    return None


def check_ds_rowsum(orc, T=8, d=4, causal=1, scale=0.45, seed=7):
    q, k, v, dO = tiny_case(seed, T, d)
    *_, ds, _ = orc.bwd_head(q, k, v, dO, scale, causal, want_ds=True)
    if np.max(np.abs(ds.sum(axis=1))) > 1e-12:
        return "rowsum(dS) != 0"
    return None


def check_zero_dO(orc, T=8, d=4, causal=1, scale=0.45, seed=8):
    q, k, v, _ = tiny_case(seed, T, d)
    dq, dk, dv = orc.bwd_head(q, k, v, np.zeros((T, d)), scale, causal)
    if np.any(dq != 0) or np.any(dk != 0) or np.any(dv != 0):
        return "dO = 0 did not give exactly zero gradients"
    return None


def check_rows_match_full(orc, T=11, d=3, causal=1, scale=0.66, seed=9):
    q, k, v, dO = tiny_case(seed, T, d)
    o, lse = orc.fwd_head(q, k, v, scale, causal)
    dq, dk, dv = orc.bwd_head(q, k, v, dO, scale, causal)
    qi, ki = [0, 4, 10], [0, 5, 10]
    ro, rl, rdq, rdk, rdv = orc.rows_head(q, k, v, dO, scale, causal, qi, ki)
    for a, b, n in ((ro, o[qi], "O"), (rl, lse[qi], "LSE"), (rdq, dq[qi], "dQ"),
                    (rdk, dk[ki], "dK"), (rdv, dv[ki], "dV")):
        if np.max(np.abs(a - b)) > 1e-12:
            return f"row-sampled {n} differs from the full oracle"
    return None


def _golden_eval(expr: str) -> float:
    return float(eval(expr, {"__builtins__": {}}, {"log": math.log}))


def _golden_split(rhs: str):
    # entries are separated by commas outside parentheses
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
    return [_golden_eval(e.strip()) for e in out if e.strip()]


def golden_fixtures():
    return sorted(glob.glob(os.path.join(GOLDEN, "worked_*.txt")))


def load_golden(path):
    """A worked example: {name: array}; "name = ..." is a vector, "name[i] = ..."
    row i of a matrix; entries are exact expressions (log = natural log)."""
    vec, mat = {}, {}
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            lhs, rhs = (x.strip() for x in line.split("=", 1))
            vals = _golden_split(rhs)
            if "[" in lhs:
                name, idx = lhs[:-1].split("[")
                mat.setdefault(name, {})[int(idx)] = vals
            else:
                vec[lhs] = vals
    for name, rows in mat.items():
        vec[name] = [rows[i] for i in range(len(rows))]
    return {k: np.array(v, dtype=np.float64) for k, v in vec.items()}


def check_worked_examples(orc, tol=1e-13):
    """The oracle's P, LSE, O, D, dS, dV, dK, dQ against every worked example."""
    paths = golden_fixtures()
    if not paths:
        return "no worked examples found"
    for path in paths:
        fx = load_golden(path)
        scale, causal = float(fx["scale"][0]), int(fx["causal"][0])
        q, k, v, dO = (fx[n].reshape(-1, 1) for n in ("q", "k", "v", "dO"))
        o, lse, p = orc.fwd_head(q, k, v, scale, causal, want_p=True)
        dq, dk, dv, ds, dvec = orc.bwd_head(q, k, v, dO, scale, causal, want_ds=True)
        got = {"p": p, "lse": lse, "o": o[:, 0], "D": dvec, "ds": ds, "dv": dv[:, 0],
               "dk": dk[:, 0], "dq": dq[:, 0]}
        for name, value in got.items():
            err = float(np.max(np.abs(value - fx[name])))
            if not err <= tol:
                return f"worked example {os.path.basename(path)}: {name} off by {err:.3g}"
    return None


def all_checks(orc):
    """Run every pin; return the list of failure messages (empty when all pass)."""
    out = []
    for fn, kw in [
        (check_brute_force, dict(causal=1)),
        (check_brute_force, dict(causal=0, T=5, d=3, scale=1.3)),
        (check_brute_force, dict(causal=1, T=8, d=64, scale=0.125)),
        (check_finite_differences, dict(causal=1)),
        (check_finite_differences, dict(causal=0, T=5, d=3, scale=1.1)),
        (check_zero_q_closed_form, dict(causal=1)),
        (check_zero_q_closed_form, dict(causal=0)),
        (check_t1_closed_form, {}),
        (check_softmax_rows, {}),
        (check_causal_independence, {}),
        (check_ds_rowsum, {}),
        (check_zero_dO, {}),
        (check_rows_match_full, dict(causal=1)),
        (check_rows_match_full, dict(causal=0)),
        (check_worked_examples, {}),
    ]:
        try:
            msg = fn(orc, **kw)
        except Exception as e:  # a crash in a mutated oracle is a failed pin too
            msg = f"{fn.__name__}: raised {e!r}"
        if msg:
            out.append(msg)
    return out
