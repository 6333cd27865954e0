"""Pins of the fp64 softmax-anchor oracle (oracle/gla_softmax_oracle.py).

What each check pins:
  * the mask, against torch's scaled_dot_product_attention (a library
    routine) given the boolean mask built independently, element by element
    from frame indices: window edges, sinks, no double counting;
  * one frame with a window of one: plain full (non-causal) attention;
  * a window covering every frame without sinks: block-causal attention;
  * constant values: every softmax row sums to one, so out = v;
  * the output gate: sigmoid(z) elementwise, and gate logits of +inf leave
    the attention output unchanged;
  * planted mistakes (window one frame short, sinks counted twice, no 1/sqrt(d)
    scale, gate applied before the attention), each caught.
"""

import numpy as np
import pytest
import torch

from oracle.gla_softmax_oracle import anchor_key_ranges, softmax_anchor_head


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def sdpa_reference(q, k, v, T, window, n_sink):
    """torch SDPA with a mask written from the frame of each query and key."""
    n, d = q.shape
    fq = np.arange(n)[:, None] // T
    fk = np.arange(n)[None, :] // T
    in_window = (fk <= fq) & (fk >= fq - window + 1)
    is_sink = (np.arange(n)[None, :] < n_sink) & (fk <= fq)  # sinks never reach the future
    mask = torch.from_numpy(in_window | is_sink)
    t = lambda x: torch.from_numpy(x)[None, None]  # noqa: E731
    out = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=mask[None, None])
    return out[0, 0].numpy()


CASES = [  # F, T, d, window, n_sink
    (4, 6, 8, 1, 0),
    (4, 6, 8, 2, 0),
    (5, 5, 16, 2, 3),
    (5, 4, 8, 3, 4),     # sinks = the whole first frame
    (6, 3, 8, 2, 7),     # sinks reach into frame 2
    (3, 7, 8, 5, 2),     # window larger than the sequence
]


@pytest.mark.parametrize("F,T,d,window,n_sink", CASES)
def test_matches_masked_sdpa(F, T, d, window, n_sink):
    q, k, v = rnd((F * T, d), 1 + d), rnd((F * T, d), 2 + d), rnd((F * T, d), 3 + d)
    out = softmax_anchor_head(q, k, v, T, window, n_sink)
    np.testing.assert_allclose(out, sdpa_reference(q, k, v, T, window, n_sink), rtol=1e-10,
                               atol=1e-12)


def test_key_ranges_are_disjoint_and_cover_the_mask():
    for f in range(6):
        (s0, s1), (w0, w1) = anchor_key_ranges(f, 5, 2, 7)
        assert s1 <= w0 and s0 == 0 and w1 == (f + 1) * 5
        assert w0 == max(0, f - 1) * 5
        assert s1 == min(7, w0)


def test_single_frame_is_full_attention():
    T, d = 9, 16
    q, k, v = rnd((T, d), 5), rnd((T, d), 6), rnd((T, d), 7)
    s = q @ k.T / np.sqrt(d)
    p = np.exp(s - s.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    np.testing.assert_allclose(softmax_anchor_head(q, k, v, T, 1, 0), p @ v, rtol=1e-12)


def test_constant_values_pass_through():
    F, T, d = 4, 5, 8
    q, k = rnd((F * T, d), 8), rnd((F * T, d), 9)
    v = np.tile(rnd((1, d), 10), (F * T, 1))
    np.testing.assert_allclose(softmax_anchor_head(q, k, v, T, 2, 3), v, rtol=1e-12)


def test_output_gate():
    F, T, d = 3, 4, 8
    q, k, v, z = (rnd((F * T, d), s) for s in (11, 12, 13, 14))
    plain = softmax_anchor_head(q, k, v, T, 2, 2)
    gated = softmax_anchor_head(q, k, v, T, 2, 2, z)
    np.testing.assert_allclose(gated, plain / (1 + np.exp(-z)), rtol=1e-12)
    np.testing.assert_allclose(softmax_anchor_head(q, k, v, T, 2, 2, np.full_like(z, np.inf)),
                               plain, rtol=1e-12)


def _planted(kind, q, k, v, T, window, n_sink, z=None):
    n, d = q.shape
    out = np.zeros((n, d))
    for f in range(n // T):
        w_lo = max(0, f - window + (2 if kind == "short_window" else 1)) * T
        w_hi = (f + 1) * T
        sinks = np.arange(min(n_sink, w_lo) if kind != "double_sinks" else n_sink)
        keys = np.r_[sinks, np.arange(w_lo, w_hi)]
        rows = slice(f * T, (f + 1) * T)
        scale = 1.0 if kind == "no_scale" else 1.0 / np.sqrt(d)
        qq = q[rows] * (1 / (1 + np.exp(-z[rows])) if kind == "gate_first" else 1.0)
        s = qq @ k[keys].T * scale
        p = np.exp(s - s.max(1, keepdims=True))
        p /= p.sum(1, keepdims=True)
        out[rows] = p @ v[keys]
    if kind != "gate_first" and z is not None:
        out /= 1 + np.exp(-z)
    return out


@pytest.mark.parametrize("kind", ["short_window", "double_sinks", "no_scale", "gate_first"])
def test_planted_mistakes_are_caught(kind):
    F, T, d, window, n_sink = 5, 5, 8, 2, 4
    q, k, v, z = (rnd((F * T, d), s) for s in (21, 22, 23, 24))
    bad = _planted(kind, q, k, v, T, window, n_sink, z)
    good = softmax_anchor_head(q, k, v, T, window, n_sink, z)
    assert np.abs(bad - good).max() > 1e-3
    ref = sdpa_reference(q, k, v, T, window, n_sink) / (1 + np.exp(-z))
    np.testing.assert_allclose(good, ref, rtol=1e-10, atol=1e-12)
