"""Pins of the fp64 AdamW oracle (CPU).  None re-types the oracle's formulas: the
reference points are torch.optim.AdamW in float64 (its update is the same AdamW with
epsilon outside the square root and decoupled weight decay), a closed form of the
first step from zero moments, brute-force norms, and the clip's defining property."""
import math

import numpy as np
import pytest
import torch

from oracle import adamw as oa

HP = dict(lr=3e-3, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1)


def _state(seed, shapes):
    rng = np.random.default_rng(seed)
    ps = [rng.normal(0, 0.5, s) for s in shapes]
    gs = [rng.normal(0, 0.3, s) for s in shapes]
    return ps, gs


SHAPES = [(7, 5), (13,), (3, 4, 2), (1,), (64, 3)]
DECAY = [len(s) >= 2 for s in SHAPES]


def test_matches_torch_adamw_over_several_steps():
    ps, _ = _state(0, SHAPES)
    tp = [torch.tensor(p, dtype=torch.float64, requires_grad=True) for p in ps]
    groups = [{"params": [t for t, d in zip(tp, DECAY) if d], "weight_decay": HP["weight_decay"]},
              {"params": [t for t, d in zip(tp, DECAY) if not d], "weight_decay": 0.0}]
    opt = torch.optim.AdamW(groups, lr=HP["lr"], betas=(HP["beta1"], HP["beta2"]),
                            eps=HP["eps"])
    ms = [np.zeros(s) for s in SHAPES]
    vs = [np.zeros(s) for s in SHAPES]
    cur = [p.copy() for p in ps]
    for step in range(1, 5):
        _, gs = _state(100 + step, SHAPES)
        for t, g in zip(tp, gs):
            t.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
        cur, ms, vs, _ = oa.adamw_step(cur, gs, ms, vs, DECAY, step=step, max_norm=0.0, **HP)
        for a, t in zip(cur, tp):
            np.testing.assert_allclose(a, t.detach().numpy(), rtol=1e-12, atol=1e-15)


def test_first_step_from_zero_moments_closed_form():
    # m^ = g and v^ = g^2 at step 1, so the update is g / (|g| + eps) + wd p
    ps, gs = _state(1, SHAPES)
    zeros = [np.zeros(s) for s in SHAPES]
    new, m, v, _ = oa.adamw_step(ps, gs, zeros, zeros, DECAY, step=1, max_norm=0.0, **HP)
    for p, g, n, d in zip(ps, gs, new, DECAY):
        wd = HP["weight_decay"] if d else 0.0
        want = p - HP["lr"] * (g / (np.abs(g) + HP["eps"]) + wd * p)
        np.testing.assert_allclose(n, want, rtol=1e-13, atol=1e-16)


def test_zero_gradient_leaves_only_the_decay():
    ps, _ = _state(2, SHAPES)
    zeros = [np.zeros(s) for s in SHAPES]
    new, m, v, norm = oa.adamw_step(ps, zeros, zeros, zeros, DECAY, step=3, max_norm=1.0, **HP)
    assert norm == 0.0
    for p, n, d in zip(ps, new, DECAY):
        f = 1 - HP["lr"] * HP["weight_decay"] if d else 1.0
        np.testing.assert_allclose(n, p * f, rtol=1e-15)


def test_global_norm_is_brute_force_norm():
    _, gs = _state(3, SHAPES)
    want = math.sqrt(math.fsum(float(x) ** 2 for g in gs for x in np.ravel(g)))
    assert oa.global_norm(gs) == pytest.approx(want, rel=1e-14)


def test_clip_is_the_unclipped_step_on_scaled_gradients():
    ps, gs = _state(4, SHAPES)
    ms = [np.full(s, 0.01) for s in SHAPES]
    vs = [np.full(s, 0.02) for s in SHAPES]
    norm = oa.global_norm(gs)
    max_norm = 0.25 * norm
    a = oa.adamw_step(ps, gs, ms, vs, DECAY, step=5, max_norm=max_norm, **HP)
    scaled = [g * (max_norm / norm) for g in gs]
    b = oa.adamw_step(ps, scaled, ms, vs, DECAY, step=5, max_norm=0.0, **HP)
    for x, y in zip(a[0] + a[1] + a[2], b[0] + b[1] + b[2]):
        np.testing.assert_allclose(x, y, rtol=1e-13, atol=1e-18)
    # the clipped gradients have exactly the requested norm; a large max_norm clips nothing
    assert oa.global_norm(scaled) == pytest.approx(max_norm, rel=1e-13)
    c = oa.adamw_step(ps, gs, ms, vs, DECAY, step=5, max_norm=10 * norm, **HP)
    d = oa.adamw_step(ps, gs, ms, vs, DECAY, step=5, max_norm=0.0, **HP)
    for x, y in zip(c[0], d[0]):
        assert np.array_equal(x, y)


def test_vectors_take_no_weight_decay():
    ps, gs = _state(5, SHAPES)
    zeros = [np.zeros(s) for s in SHAPES]
    a = oa.adamw_step(ps, gs, zeros, zeros, DECAY, step=1, max_norm=0.0, **HP)[0]
    hp = dict(HP, weight_decay=0.0)
    b = oa.adamw_step(ps, gs, zeros, zeros, DECAY, step=1, max_norm=0.0, **hp)[0]
    for x, y, d in zip(a, b, DECAY):
        assert np.array_equal(x, y) != d


# Plant one plausible mistake at a time in a copy of the AdamW oracle and check that
# the pins above catch each one.
MUTATIONS = {
    "eps inside the square root": ("np.sqrt(v_hat) + eps", "np.sqrt(v_hat + eps)"),
    "no bias correction of m": ("m_hat = m / bc1", "m_hat = m"),
    "decay on every tensor": ("wd = weight_decay if dec else 0.0", "wd = weight_decay"),
    "decay scaled away from lr": ("p = p - lr * (m_hat / (np.sqrt(v_hat) + eps) + wd * p)",
                                  "p = p - lr * m_hat / (np.sqrt(v_hat) + eps) - wd * p"),
    "clip factor inverted": ("return max_norm / norm if", "return norm / max_norm if"),
    "second moment from the unclipped gradient": (
        "v = beta2 * np.asarray(v, dtype=np.float64) + (1.0 - beta2) * g * g",
        "v = beta2 * np.asarray(v, dtype=np.float64) + (1.0 - beta2) * g * g / c / c"),
    "beta1 and 1 - beta1 swapped": ("m = beta1 * np.asarray(m, dtype=np.float64) + (1.0 - beta1) * g",
                                    "m = (1.0 - beta1) * np.asarray(m, dtype=np.float64) + beta1 * g"),
}
PINS = [test_matches_torch_adamw_over_several_steps, test_first_step_from_zero_moments_closed_form,
        test_zero_gradient_leaves_only_the_decay, test_global_norm_is_brute_force_norm,
        test_clip_is_the_unclipped_step_on_scaled_gradients, test_vectors_take_no_weight_decay]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_adamw_mutation(name, monkeypatch):
    import types

    src = open(oa.__file__).read()
    old, new = MUTATIONS[name]
    assert src.count(old) == 1, name
    mutant = types.ModuleType("adamw_mutant")
    exec(compile(src.replace(old, new), "adamw_mutant", "exec"), mutant.__dict__)
    caught = 0
    for pin in PINS:
        monkeypatch.setattr(pin.__globals__["oa"], "adamw_step", mutant.adamw_step)
        monkeypatch.setattr(pin.__globals__["oa"], "global_norm", mutant.global_norm)
        try:
            pin()
        except (AssertionError, ZeroDivisionError, FloatingPointError):
            caught += 1
        monkeypatch.undo()
    assert caught, f"no pin caught: {name}"
