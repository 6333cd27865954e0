"""Pins of the fp64 RoPE oracle (oracle/gla_rope_oracle.py), CPU only.

What each check pins:
  * golden angles (tests/golden/rope_angles.txt, worked by hand): the
    position of a token (frame offset, row, column), the block layout
    [temporal | height | width] and the frequency law;
  * rotation identities (zero angle, quarter turn, composition, norm): the
    pair layout and the sense of rotation;
  * zero angles reduce to the plain layer (gla_oracle.gla_head);
  * a brute-force quadratic form with the rotation written in complex
    numbers and only angle differences: the recurrence, that q and k turn by
    the same angles, and that the normaliser is left un-rotated;
  * shift invariance in the frame offset (only relative positions matter);
  * chunking through state_in / state_out with the offset advanced;
  * planted mistakes, each caught by one of the above.
"""

import os

import numpy as np
import pytest

from oracle import gla_head, gla_rope_bruteforce_head, gla_rope_head, rope_pair_angles, rope_rotate

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "rope_angles.txt")


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def test_golden_angles():
    rows = [ln.split() for ln in open(GOLDEN) if ln.strip() and not ln.startswith("#")]
    want = np.array([float(r[4]) for r in rows])
    # token t = 7 of frame f = 1, frame_offset = 3, grid_w = 5
    got = rope_pair_angles(np.array([3 + 1]), np.array([7 // 5]), np.array([7 % 5]), (8, 0, 8),
                           100.0)[0]
    np.testing.assert_allclose(got, want, rtol=1e-14, atol=1e-14)
    # the same through the layer's own position mapping: a frame of 8 tokens
    # rotated by its angles equals rotating token 7 by the golden angles
    x = rnd((8, 16), 1)
    ang_layer = rope_pair_angles(np.full(8, 4), np.arange(8) // 5, np.arange(8) % 5, (8, 0, 8),
                                 100.0)
    np.testing.assert_allclose(rope_rotate(x, ang_layer)[7], rope_rotate(x[7:8], want[None])[0],
                               rtol=1e-13)


def test_rotation_identities():
    x = rnd((5, 8), 2)
    z = np.zeros((5, 4))
    np.testing.assert_array_equal(rope_rotate(x, z), x)
    q = rope_rotate(x, np.full((5, 4), np.pi / 2))
    np.testing.assert_allclose(q[:, 0::2], -x[:, 1::2], atol=1e-15)  # (x0, x1) -> (-x1, x0)
    np.testing.assert_allclose(q[:, 1::2], x[:, 0::2], atol=1e-15)
    a, b = rnd((5, 4), 3), rnd((5, 4), 4)
    np.testing.assert_allclose(rope_rotate(rope_rotate(x, a), b), rope_rotate(x, a + b),
                               atol=1e-13)
    np.testing.assert_allclose(np.linalg.norm(rope_rotate(x, a), axis=1),
                               np.linalg.norm(x, axis=1), rtol=1e-14)


def test_zero_angles_is_the_plain_layer():
    d, T = 16, 9
    q, k, v = rnd((T, d), 5), rnd((T, d), 6), rnd((T, d), 7)
    g = np.array([1.3])
    s = rnd((d, d + 1), 8)
    s[:, d] = np.abs(s[:, d]) + 1
    o1, s1 = gla_rope_head(q, k, v, g, T, grid_w=3, frame_offset=0, dims=(16, 0, 0), state_in=s)
    # one frame at offset 0: every temporal angle is 0, and there are no
    # spatial blocks
    o0, s0 = gla_head(q, k, v, g, T, s)
    np.testing.assert_allclose(o1, o0, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s1, s0, rtol=1e-12, atol=1e-12)


CASES = [
    # d, dims, F, T, grid_w, offset, theta
    (8, (8, 0, 0), 3, 4, 2, 0, 10000.0),
    (16, (8, 0, 8), 2, 6, 3, 5, 100.0),
    (24, (8, 8, 8), 3, 5, 2, 1, 10.0),
    (32, (8, 16, 8), 2, 7, 7, 0, 10000.0),
    (16, (0, 8, 8), 4, 3, 1, 2, 3.0),
]


@pytest.mark.parametrize("d,dims,F,T,grid_w,offset,theta", CASES)
def test_bruteforce_complex_form(d, dims, F, T, grid_w, offset, theta):
    q, k, v = rnd((F * T, d), 10 + d), rnd((F * T, d), 11 + d), rnd((F * T, d), 12 + d)
    g = rnd(F, 13 + d, 1.0) + 1.0
    o, _ = gla_rope_head(q, k, v, g, T, grid_w, offset, dims, theta)
    ob = gla_rope_bruteforce_head(q, k, v, g, T, grid_w, offset, dims, theta)
    np.testing.assert_allclose(o, ob, rtol=1e-10, atol=1e-12)


def test_shift_invariance_in_frame_offset():
    d, F, T = 24, 3, 10
    q, k, v = rnd((F * T, d), 20), rnd((F * T, d), 21), rnd((F * T, d), 22)
    g = rnd(F, 23) + 2
    o0, _ = gla_rope_head(q, k, v, g, T, 4, 0, (8, 8, 8), 50.0)
    o7, _ = gla_rope_head(q, k, v, g, T, 4, 7, (8, 8, 8), 50.0)
    np.testing.assert_allclose(o0, o7, rtol=1e-9, atol=1e-12)
    # a spatial block does not commute with the frame offset in this way:
    # changing grid_w changes the result
    o5, _ = gla_rope_head(q, k, v, g, T, 5, 0, (8, 8, 8), 50.0)
    assert np.abs(o5 - o0).max() > 1e-6


def test_chunking_with_offsets():
    d, F, T = 16, 5, 6
    q, k, v = rnd((F * T, d), 30), rnd((F * T, d), 31), rnd((F * T, d), 32)
    g = rnd(F, 33) + 1
    dims, w, off = (8, 0, 8), 4, 2
    s = rnd((d, d + 1), 34)
    s[:, d] = np.abs(s[:, d]) + 1
    o, so = gla_rope_head(q, k, v, g, T, w, off, dims, 100.0, s)
    n1 = 2 * T
    oa, sa = gla_rope_head(q[:n1], k[:n1], v[:n1], g[:2], T, w, off, dims, 100.0, s)
    ob, sb = gla_rope_head(q[n1:], k[n1:], v[n1:], g[2:], T, w, off + 2, dims, 100.0, sa)
    np.testing.assert_allclose(np.vstack([oa, ob]), o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sb, so, rtol=1e-12, atol=1e-12)


def test_normaliser_column_is_unrotated():
    d, F, T = 16, 3, 5
    q, k, v = rnd((F * T, d), 40), rnd((F * T, d), 41), rnd((F * T, d), 42)
    g = rnd(F, 43)
    _, s_rope = gla_rope_head(q, k, v, g, T, 2, 3, (8, 8, 0), 100.0)
    _, s_plain = gla_head(q, k, v, g, T, None)
    np.testing.assert_allclose(s_rope[:, d], s_plain[:, d], rtol=1e-13)


# ------------------------------------------------------------ planted mistakes


def _planted(kind, q, k, v, g, T, grid_w, offset, dims, theta, eps=1e-6):
    """The recurrence with one mistake planted (CPU only)."""
    d = q.shape[1]
    S = np.zeros((d, d + 1))
    out = np.zeros_like(q)
    a_all = 1 / (1 + np.exp(-g))
    for f in range(len(g)):
        rows = slice(f * T, (f + 1) * T)
        t = np.arange(T)
        pt = np.full(T, offset + f)
        py, px = (t % grid_w, t // grid_w) if kind == "axes_swapped" else (t // grid_w, t % grid_w)
        ang = rope_pair_angles(pt, py, px, dims, theta)
        Kf = np.maximum(k[rows], 0)
        Qf = np.maximum(q[rows], 0)
        Kr = rope_rotate(Kf, -ang if kind == "k_turns_back" else ang)
        Qr = Qf if kind == "q_not_rotated" else rope_rotate(Qf, ang)
        S[:, :d] = a_all[f] * S[:, :d] + Kr.T @ v[rows]
        S[:, d] = a_all[f] * S[:, d] + (Kr if kind == "rotated_normaliser" else Kf).sum(axis=0)
        den = (Qr if kind == "rotated_normaliser" else Qf) @ S[:, d] + eps
        out[rows] = (Qr @ S[:, :d]) / den[:, None]
    return out


@pytest.mark.parametrize("kind", ["k_turns_back", "q_not_rotated", "rotated_normaliser",
                                  "axes_swapped"])
def test_planted_mistakes_are_caught(kind):
    d, F, T, w, off, dims, theta = 24, 2, 6, 4, 1, (8, 8, 8), 20.0
    q, k, v = rnd((F * T, d), 50), rnd((F * T, d), 51), rnd((F * T, d), 52)
    g = rnd(F, 53) + 1
    bad = _planted(kind, q, k, v, g, T, w, off, dims, theta)
    good = gla_rope_bruteforce_head(q, k, v, g, T, w, off, dims, theta)
    # the brute force tells the planted mistake apart from the correct
    # recurrence, which matches it
    assert np.abs(bad - good).max() > 1e-3 * np.abs(good).max()
    ok, _ = gla_rope_head(q, k, v, g, T, w, off, dims, theta)
    np.testing.assert_allclose(ok, good, rtol=1e-10, atol=1e-12)
