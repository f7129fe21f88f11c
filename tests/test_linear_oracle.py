"""Pins of the fp64 projection-GEMM oracle (CPU).  None re-types the oracle: brute
force is a triple loop summed with math.fsum, the backward products are checked as
the gradients of L = sum(dY o Y) by central differences (exact up to rounding for a
linear map) and by torch autograd in float64, and planted mistakes must be caught."""
import math
import types

import numpy as np
import pytest
import torch

from oracle import linear as ol


def _inputs(seed, t=5, i=4, o=3):
    rng = np.random.default_rng(seed)
    return rng.normal(size=(t, i)), rng.normal(size=(o, i)), rng.normal(size=(t, o))


def check_brute_force(mod):
    x, w, dy = _inputs(0)
    T, I = x.shape
    O = w.shape[0]
    y = np.array([[math.fsum(x[t, i] * w[o, i] for i in range(I)) for o in range(O)]
                  for t in range(T)])
    dx = np.array([[math.fsum(dy[t, o] * w[o, i] for o in range(O)) for i in range(I)]
                   for t in range(T)])
    dw = np.array([[math.fsum(dy[t, o] * x[t, i] for t in range(T)) for i in range(I)]
                   for o in range(O)])
    np.testing.assert_allclose(mod.linear_fwd(x, w), y, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(mod.linear_bwd_dx(dy, w), dx, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(mod.linear_bwd_dw(dy, x), dw, rtol=1e-13, atol=1e-14)


def check_finite_differences(mod):
    x, w, dy = _inputs(1, 4, 3, 2)
    h = 1e-6

    def loss(xx, ww):
        return float(np.sum(dy * mod.linear_fwd(xx, ww)))

    gx = np.zeros_like(x)
    for idx in np.ndindex(*x.shape):
        e = np.zeros_like(x)
        e[idx] = h
        gx[idx] = (loss(x + e, w) - loss(x - e, w)) / (2 * h)
    gw = np.zeros_like(w)
    for idx in np.ndindex(*w.shape):
        e = np.zeros_like(w)
        e[idx] = h
        gw[idx] = (loss(x, w + e) - loss(x, w - e)) / (2 * h)
    np.testing.assert_allclose(mod.linear_bwd_dx(dy, w), gx, rtol=1e-7, atol=1e-8)
    np.testing.assert_allclose(mod.linear_bwd_dw(dy, x), gw, rtol=1e-7, atol=1e-8)


def check_torch_autograd(mod):
    x, w, dy = _inputs(2, 17, 9, 6)
    tx = torch.tensor(x, requires_grad=True)
    tw = torch.tensor(w, requires_grad=True)
    y = torch.nn.functional.linear(tx, tw)
    y.backward(torch.tensor(dy))
    np.testing.assert_allclose(mod.linear_fwd(x, w), y.detach().numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(mod.linear_bwd_dx(dy, w), tx.grad.numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(mod.linear_bwd_dw(dy, x), tw.grad.numpy(), rtol=1e-12, atol=1e-13)


CHECKS = [check_brute_force, check_finite_differences, check_torch_autograd]


@pytest.mark.parametrize("check", CHECKS, ids=[c.__name__ for c in CHECKS])
def test_oracle_pins(check):
    check(ol)


MUTATIONS = {
    "forward with the rows of W reversed": (
        "return np.asarray(x, dtype=np.float64) @ np.asarray(w, dtype=np.float64).T",
        "return np.asarray(x, dtype=np.float64) @ np.asarray(w, dtype=np.float64)[::-1].T"),
    "dX with one output feature dropped": (
        "return np.asarray(dy, dtype=np.float64) @ np.asarray(w, dtype=np.float64)",
        "return np.asarray(dy, dtype=np.float64)[:, 1:] @ np.asarray(w, dtype=np.float64)[1:]"),
    "dW summed over one token fewer": (
        "return np.asarray(dy, dtype=np.float64).T @ np.asarray(x, dtype=np.float64)",
        "return np.asarray(dy, dtype=np.float64)[:-1].T @ np.asarray(x, dtype=np.float64)[:-1]"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_linear_mutation(name):
    src = open(ol.__file__).read()
    old, new = MUTATIONS[name]
    assert src.count(old) == 1, name
    mutant = types.ModuleType("linear_mutant")
    exec(compile(src.replace(old, new), "linear_mutant", "exec"), mutant.__dict__)
    caught = 0
    for check in CHECKS:
        try:
            check(mutant)
        except (AssertionError, ValueError):
            caught += 1
    assert caught, f"no pin caught: {name}"
