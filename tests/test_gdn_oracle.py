"""Pins of the fp64 frame-wise gated delta-rule oracle (oracle/gla_gdn_oracle.py).

What each check pins:
  * beta = 0: the state only decays (a pure gated scan of state_in, the
    queries reading a_0 ... a_f state_in);
  * one frame from the zero state: the base layer's output (the write is
    beta K~^T V1 and beta cancels in the ratio when eps = 0);
  * the delta rule's defining property: keys with orthonormal rows
    (one-hot, so ReLU keeps them) and beta = a = 1 read back exactly the
    frame's values, whatever the state held before;
  * the fixed point: frames that repeat the same keys and values drive the
    state to the solution of S = a (I - beta M) S + beta K~^T V1 (a library
    linear solve), with M = K~^T K~;
  * chunking through state_in / state_out;
  * planted mistakes (no decay inside the correction, the Gram matrix of the
    wrong side, the correction's sign), each caught by one of the above.
"""

import numpy as np
import pytest

from oracle import gla_head
from oracle.gla_gdn_oracle import gla_gdn_head


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def test_beta_zero_only_decays():
    d, F, T = 16, 4, 5
    q, k, v = rnd((F * T, d), 1), rnd((F * T, d), 2), rnd((F * T, d), 3)
    g = rnd(F, 4) + 1
    s = rnd((d, d + 1), 5)
    s[:, d] = np.abs(s[:, d]) + 1
    out, so = gla_gdn_head(q, k, v, g, np.full(F, -np.inf), T, s)
    a = 1 / (1 + np.exp(-g))
    np.testing.assert_allclose(so, np.prod(a) * s, rtol=1e-13)
    Q = np.maximum(q, 0)
    for f in range(F):
        Sf = np.prod(a[: f + 1]) * s
        rows = slice(f * T, (f + 1) * T)
        want = (Q[rows] @ Sf[:, :d]) / (Q[rows] @ Sf[:, d] + 1e-6)[:, None]
        np.testing.assert_allclose(out[rows], want, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("beta_logit", [-1.0, 0.0, 2.5])
def test_first_frame_from_zero_state_is_the_base_layer(beta_logit):
    d, T = 24, 9
    q, k, v = rnd((T, d), 10), rnd((T, d), 11), rnd((T, d), 12)
    g = np.array([0.7])
    out, _ = gla_gdn_head(q, k, v, g, np.array([beta_logit]), T, None, eps=0.0)
    base, _ = gla_head(q, k, v, g, T, None, 0.0)
    np.testing.assert_allclose(out, base, rtol=1e-11, atol=1e-12)


def test_orthonormal_keys_read_back_their_values():
    d, T = 16, 6
    rng = np.random.default_rng(20)
    idx = rng.permutation(d)[:T]
    k = np.zeros((2 * T, d))
    k[T + np.arange(T), idx] = 1.0          # frame 1: one-hot keys, orthonormal rows
    k[:T] = rnd((T, d), 21)                 # frame 0: anything
    v = rnd((2 * T, d), 22)
    q = k.copy()                             # frame 1's queries equal its keys
    s = rnd((d, d + 1), 23)
    g = np.array([0.3, np.inf])              # a_1 = 1
    bl = np.array([0.2, np.inf])             # beta_1 = 1
    out, S = gla_gdn_head(q, k, v, g, bl, T, s, eps=0.0)
    K1 = k[T:]
    np.testing.assert_allclose(K1 @ S[:, :d], v[T:], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(K1 @ S[:, d], np.ones(T), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out[T:], v[T:], rtol=1e-12, atol=1e-12)


def test_repeated_frame_reaches_the_fixed_point():
    d, T, F = 8, 20, 400
    k1 = rnd((T, d), 30, 1 / np.sqrt(d * T))   # the pages' 1/sqrt(D S) key scale
    v1 = rnd((T, d), 31)
    k = np.tile(k1, (F, 1))
    v = np.tile(v1, (F, 1))
    q = rnd((F * T, d), 32)
    g = np.full(F, 1.5)
    bl = np.full(F, 0.4)
    _, S = gla_gdn_head(q, k, v, g, bl, T, None)
    a, beta = 1 / (1 + np.exp(-1.5)), 1 / (1 + np.exp(-0.4))
    K = np.maximum(k1, 0)
    M = K.T @ K
    A = a * (np.eye(d) - beta * M)
    rhs = beta * K.T @ np.hstack([v1, np.ones((T, 1))])
    S_star = np.linalg.solve(np.eye(d) - A, rhs)
    np.testing.assert_allclose(S, S_star, rtol=1e-9, atol=1e-12)


def test_chunking_invariance():
    d, F, T = 16, 5, 7
    q, k, v = rnd((F * T, d), 40), rnd((F * T, d), 41, 0.3), rnd((F * T, d), 42)
    g, bl = rnd(F, 43) + 1, rnd(F, 44)
    s = rnd((d, d + 1), 45)
    s[:, d] = np.abs(s[:, d]) + 1
    o, so = gla_gdn_head(q, k, v, g, bl, T, s)
    n = 2 * T
    oa, sa = gla_gdn_head(q[:n], k[:n], v[:n], g[:2], bl[:2], T, s)
    ob, sb = gla_gdn_head(q[n:], k[n:], v[n:], g[2:], bl[2:], T, sa)
    np.testing.assert_allclose(np.vstack([oa, ob]), o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sb, so, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------ planted mistakes


def _planted(kind, q, k, v, g, bl, T, s, eps=0.0):
    d = q.shape[1]
    S = np.zeros((d, d + 1)) if s is None else s.copy()
    out = np.zeros_like(q)
    for f in range(len(g)):
        rows = slice(f * T, (f + 1) * T)
        a, beta = 1 / (1 + np.exp(-g[f])), 1 / (1 + np.exp(-bl[f]))
        K = np.maximum(k[rows], 0)
        V1 = np.hstack([v[rows], np.ones((T, 1))])
        if kind == "undecayed_read":
            S = a * S + beta * K.T @ (V1 - K @ S)
        elif kind == "plus_sign":
            S = a * S + beta * K.T @ (V1 + a * K @ S)
        elif kind == "gram_after":  # the correction multiplies the state from the right
            M = K.T @ K
            Sv = a * (S[:, :d] - beta * S[:, :d] @ M) + beta * K.T @ v[rows]
            Sz = a * (S[:, d] - beta * M @ S[:, d]) + beta * K.sum(axis=0)
            S = np.hstack([Sv, Sz[:, None]])
        Q = np.maximum(q[rows], 0)
        out[rows] = (Q @ S[:, :d]) / (Q @ S[:, d] + eps)[:, None]
    return out, S


@pytest.mark.parametrize("kind", ["undecayed_read", "plus_sign", "gram_after"])
def test_planted_mistakes_are_caught(kind):
    # the orthonormal-keys pin with a < 1 and a random earlier state
    d, T = 16, 6
    rng = np.random.default_rng(50)
    idx = rng.permutation(d)[:T]
    k = rnd((2 * T, d), 51)
    k[T:] = 0.0
    k[T + np.arange(T), idx] = 1.0
    v = rnd((2 * T, d), 52)
    q = k.copy()
    s = rnd((d, d + 1), 53)
    g, bl = np.array([0.3, 0.8]), np.array([0.2, np.inf])
    _, S_bad = _planted(kind, q, k, v, g, bl, T, s)
    _, S_ok = gla_gdn_head(q, k, v, g, bl, T, s, eps=0.0)
    K1 = k[T:]
    # beta = 1, orthonormal keys: the read-back equals the values for any a
    np.testing.assert_allclose(K1 @ S_ok[:, :d], v[T:], rtol=1e-12, atol=1e-12)
    assert np.abs(K1 @ S_bad[:, :d] - v[T:]).max() > 1e-3
