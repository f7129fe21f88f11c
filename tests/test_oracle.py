"""The fp64 oracle against brute force, finite differences, closed forms,
invariants and a library routine (CPU only)."""
import math

import numpy as np
import pytest
import torch

import oracle
from tests import oracle_pins as pins


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("T,d", [(1, 1), (2, 1), (5, 4), (8, 64), (8, 1)])
def test_brute_force(orc, T, d, causal):
    for scale in (0.125, 0.9, 2.0):
        assert pins.check_brute_force(orc, T=T, d=d, causal=causal, scale=scale,
                                      seed=T * 10 + d) is None


@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("T,d,scale", [(1, 4, 0.5), (4, 1, 1.7), (6, 4, 0.61), (8, 3, 0.2)])
def test_finite_differences(orc, T, d, scale, causal):
    assert pins.check_finite_differences(orc, T=T, d=d, causal=causal, scale=scale,
                                         seed=T + d) is None


def test_finite_differences_d64(orc):
    # the workloads' head width, on a tiny sequence
    assert pins.check_finite_differences(orc, T=4, d=64, causal=1, scale=0.125) is None


@pytest.mark.parametrize("causal", [0, 1])
def test_zero_q(orc, causal):
    assert pins.check_zero_q_closed_form(orc, causal=causal) is None


def test_t1(orc):
    assert pins.check_t1_closed_form(orc) is None


@pytest.mark.parametrize("causal", [0, 1])
def test_softmax_rows(orc, causal):
    assert pins.check_softmax_rows(orc, causal=causal) is None


def test_causal_independence(orc):
    for i0 in (0, 3, 6):
        assert pins.check_causal_independence(orc, i0=i0) is None


@pytest.mark.parametrize("causal", [0, 1])
def test_ds_rowsum(orc, causal):
    assert pins.check_ds_rowsum(orc, causal=causal) is None


def test_zero_dO(orc):
    assert pins.check_zero_dO(orc) is None


@pytest.mark.parametrize("causal", [0, 1])
def test_rows_match_full(orc, causal):
    assert pins.check_rows_match_full(orc, causal=causal) is None


def _sdpa_reference(q, k, v, dO, scale, causal):
    """torch's scaled_dot_product_attention in CPU float64 with autograd."""
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, is_causal=bool(causal), scale=scale)
    o.backward(torch.tensor(dO, dtype=torch.float64))
    s = scale * (tq.detach() @ tk.detach().transpose(-1, -2))
    if causal:
        T = q.shape[-2]
        s = s.masked_fill(torch.ones(T, T, dtype=torch.bool).triu(1), float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    return (o.detach().numpy(), lse.numpy(), tq.grad.numpy(), tk.grad.numpy(),
            tv.grad.numpy())


@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("T", [1, 7, 65, 128, 200])
def test_against_torch_sdpa(orc, T, causal):
    from causal_attention_fwd_attn_b200 import workloads as wl

    w = wl.custom(1, 2, T, 64, causal=causal)
    x = {n: t.double().numpy() for n, t in wl.make_inputs(0, w, seed_offset=T).items()}
    scale = w.scale
    o, lse = orc.fwd(x["q"], x["k"], x["v"], scale, causal)
    dq, dk, dv = orc.bwd(x["q"], x["k"], x["v"], x["dO"], scale, causal)
    ro, rl, rdq, rdk, rdv = _sdpa_reference(x["q"], x["k"], x["v"], x["dO"], scale, causal)
    for a, b in ((o, ro), (lse, rl), (dq, rdq), (dk, rdk), (dv, rdv)):
        assert np.max(np.abs(a - b)) <= 1e-10 * max(1.0, np.max(np.abs(b)))


def test_tiny_workload_against_torch_sdpa(orc):
    """The tiny workload (B=1 H=2 T=128 d=64) end to end."""
    from causal_attention_fwd_attn_b200 import workloads as wl

    w = wl.WORKLOADS[0]
    x = {n: t.double().numpy() for n, t in wl.make_inputs(0).items()}
    o, lse = orc.fwd(x["q"], x["k"], x["v"], w.scale, 1)
    dq, dk, dv = orc.bwd(x["q"], x["k"], x["v"], x["dO"], w.scale, 1)
    ro, rl, rdq, rdk, rdv = _sdpa_reference(x["q"], x["k"], x["v"], x["dO"], w.scale, 1)
    for a, b in ((o, ro), (lse, rl), (dq, rdq), (dk, rdk), (dv, rdv)):
        assert np.max(np.abs(a - b)) <= 1e-10


def test_large_logits_stable(orc):
    """Scores far outside exp's range: the max-shifted softmax stays finite."""
    rng = np.random.default_rng(11)
    T, d = 16, 8
    q, k, v = (rng.standard_normal((T, d)) * 40 for _ in range(3))
    o, lse = orc.fwd_head(q, k, v, 1.0, 1)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    # each row's output is a convex combination of the allowed values
    for i in range(T):
        assert np.all(o[i] <= v[:i + 1].max(axis=0) + 1e-9)
        assert np.all(o[i] >= v[:i + 1].min(axis=0) - 1e-9)


def test_every_pin_passes(orc):
    assert pins.all_checks(orc) == []


def test_workload_inputs_are_seeded():
    from causal_attention_fwd_attn_b200 import workloads as wl

    a = wl.make_inputs(0)
    b = wl.make_inputs(0)
    for n in a:
        assert a[n].dtype == torch.bfloat16
        assert torch.equal(a[n], b[n])
        assert a[n].shape == (1, 2, 128, 64)
    assert not torch.equal(a["q"], a["k"])
    # bf16 values are exact in fp64, so both sides see the same numbers
    assert torch.equal(a["q"].double().to(torch.bfloat16), a["q"])


def test_workload_flop_counts():
    from causal_attention_fwd_attn_b200 import workloads as wl

    w = wl.WORKLOADS[1]
    assert w.flops_fwd() == 2 * 96 * 1024 * 1024 * 64
    assert math.isclose(w.flops_total() / 1e9, 45.097, rel_tol=1e-4)
