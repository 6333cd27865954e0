"""Pins for the fp64 gradient oracle: central finite differences of the
numpy forward oracle (an implementation independent of both gradient
routines), agreement of autograd with the hand-written chain rule, and
special cases (gates at +-inf give zero gate gradient; no frames passes the
state gradient through)."""

import numpy as np
import pytest
import torch

from oracle import gla_backward_head, gla_backward_head_manual, gla_forward_torch_head, gla_head


def _case(seed, F, T, d, state=True):
    r = np.random.default_rng(seed)
    N = F * T

    def away_from_zero(x):  # keep ReLU inputs off the kink for finite differences
        return np.where(np.abs(x) < 0.05, 0.05 * np.sign(x + 1e-12) + x, x)

    q = away_from_zero(r.standard_normal((N, d)))
    k = away_from_zero(r.standard_normal((N, d)))
    v = r.standard_normal((N, d))
    g = r.normal(1.0, 1.0, F)
    s = None
    if state:
        s = r.standard_normal((d, d + 1))
        s[:, d] = np.abs(s[:, d]) + 1.0
    dout = r.standard_normal((N, d))
    ds_out = r.standard_normal((d, d + 1)) if state else None
    return q, k, v, g, s, dout, ds_out


def _loss(q, k, v, g, s, dout, ds_out, T, eps):
    out, so = gla_head(q, k, v, g, T, s, eps)
    val = float(np.sum(out * dout))
    if ds_out is not None:
        val += float(np.sum(so * ds_out))
    return val


@pytest.mark.parametrize("seed,F,T,d,state", [(1, 3, 4, 4, True), (2, 2, 5, 8, False),
                                              (3, 4, 3, 6, True), (4, 1, 7, 5, True)])
def test_finite_differences(seed, F, T, d, state):
    q, k, v, g, s, dout, ds_out = _case(seed, F, T, d, state)
    eps = 1e-6
    grads = gla_backward_head_manual(q, k, v, g, T, dout, s, ds_out, eps)
    r = np.random.default_rng(100 + seed)
    inputs = [q, k, v, g] + ([s] if state else [])
    h = 1e-6
    for idx, x in enumerate(inputs):
        for _ in range(3):
            e = r.standard_normal(x.shape)
            xp, xm = x + h * e, x - h * e
            args_p = list(inputs)
            args_m = list(inputs)
            args_p[idx], args_m[idx] = xp, xm
            if not state:
                args_p.append(None)
                args_m.append(None)
            fd = (_loss(*args_p, dout, ds_out, T, eps) - _loss(*args_m, dout, ds_out, T, eps)) / (2 * h)
            an = float(np.sum(grads[idx] * e))
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (idx, fd, an)


@pytest.mark.parametrize("seed,F,T,d,state", [(5, 3, 6, 8, True), (6, 5, 2, 4, False),
                                              (7, 1, 9, 16, True)])
def test_autograd_matches_chain_rule(seed, F, T, d, state):
    q, k, v, g, s, dout, ds_out = _case(seed, F, T, d, state)
    a = gla_backward_head(q, k, v, g, T, dout, s, ds_out)
    m = gla_backward_head_manual(q, k, v, g, T, dout, s, ds_out)
    for x, y in zip(a, m):
        if x is None:
            assert y is None
            continue
        np.testing.assert_allclose(x, y, rtol=1e-10, atol=1e-11)


def test_torch_forward_matches_numpy_oracle():
    q, k, v, g, s, _, _ = _case(8, 4, 5, 8, True)
    out_t, s_t = gla_forward_torch_head(*(torch.tensor(x) for x in (q, k, v, g)), 5, torch.tensor(s))
    out_n, s_n = gla_head(q, k, v, g, 5, s)
    np.testing.assert_allclose(out_t.numpy(), out_n, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(s_t.numpy(), s_n, rtol=1e-13, atol=1e-13)


def test_saturated_gates_have_zero_gate_gradient():
    q, k, v, g, s, dout, ds_out = _case(9, 3, 4, 4, True)
    g = np.array([np.inf, -np.inf, np.inf])
    dq, dk, dv, dg, ds = gla_backward_head_manual(q, k, v, g, 4, dout, s, ds_out)
    assert np.all(dg == 0.0)
    # a_1 = 0 cuts the chain: state_in gets no gradient through frames >= 1, and
    # with a_0 = 1 it receives exactly G_0
    assert np.all(np.isfinite(ds))


def test_no_frames_passes_state_gradient_through():
    d = 4
    s = np.random.default_rng(0).standard_normal((d, d + 1))
    ds_out = np.random.default_rng(1).standard_normal((d, d + 1))
    e = np.zeros((0, d))
    r = gla_backward_head_manual(e, e, e, np.zeros(0), 0, e, s, ds_out)
    np.testing.assert_array_equal(r[4], ds_out)
