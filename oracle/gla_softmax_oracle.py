"""fp64 CPU oracle of the softmax anchor layer (attention sinks + local temporal window).

TEST INFRASTRUCTURE ONLY (like gla_oracle.py): used by the tests and the
benchmark's CPU legs, never by the library; imports nothing from the library.

The SANA-Video 2.0 pages place periodic gated-softmax anchors among the
linear layers (one in four); the SANA-WM pages add attention-sink tokens and
local temporal windows to the softmax layers for long rollouts, so that their
memory and per-chunk latency stay constant.  No formula is printed; the
reading fixed here, per (batch, head), frames f = 0..F-1 of T tokens:

  keys of a query of frame f = the tokens of frames max(0, f-W+1) .. f
                               (all of them: bidirectional inside the frame,
                               block-causal across frames, as the linear layers)
                             + the first n_sink tokens of the sequence (sinks)
                               that precede the window (so never a future
                               frame), each key counted once
  o_t   = sum_s softmax_s(q_t . k_s / sqrt(d)) v_s
  out_t = sigmoid(z_t) * o_t      (elementwise output gate; z = None: no gate)

The pins are in tests/test_softmax_oracle.py.
"""

from __future__ import annotations

import numpy as np

__all__ = ["anchor_key_ranges", "softmax_anchor_head", "softmax_anchor_forward"]


def _f64(x):
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def anchor_key_ranges(f, T, window, n_sink):
    """Token ranges [lo, hi) attended by the queries of frame f: the sink
    range (possibly empty) and the window range, disjoint."""
    w_lo = max(0, f - window + 1) * T
    w_hi = (f + 1) * T
    s_hi = min(n_sink, w_lo)  # sink tokens not already inside the window
    return (0, s_hi), (w_lo, w_hi)


def softmax_anchor_head(q, k, v, T, window, n_sink=0, z=None):
    """One (batch, head) slice: q, k, v [F*T, d] (z same shape or None)."""
    q, k, v = (_f64(x) for x in (q, k, v))
    n, d = q.shape
    F = n // T if T else 0
    out = np.zeros((n, d))
    scale = 1.0 / np.sqrt(d)
    for f in range(F):
        (s_lo, s_hi), (w_lo, w_hi) = anchor_key_ranges(f, T, window, n_sink)
        keys = np.r_[np.arange(s_lo, s_hi), np.arange(w_lo, w_hi)]
        rows = slice(f * T, (f + 1) * T)
        s = (q[rows] @ k[keys].T) * scale
        s -= s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        out[rows] = p @ v[keys]
    if z is not None:
        out *= 1.0 / (1.0 + np.exp(-_f64(z)))
    return out


def softmax_anchor_forward(q, k, v, frames, window, n_sink=0, z=None):
    """Whole batch: q, k, v (and z) [B, F*T, H, d]."""
    q, k, v = (_f64(x) for x in (q, k, v))
    zz = None if z is None else _f64(z)
    B, N, H, d = q.shape
    T = N // frames if frames else 0
    out = np.zeros_like(q)
    for b in range(B):
        for h in range(H):
            out[b, :, h] = softmax_anchor_head(q[b, :, h], k[b, :, h], v[b, :, h], T, window,
                                               n_sink, None if zz is None else zz[b, :, h])
    return out
