"""fp64 CPU oracle of the frame-wise gated delta-rule layer (Gated DeltaNet).

TEST INFRASTRUCTURE ONLY (like gla_oracle.py): used by the tests and the
benchmark's CPU legs, never by the library; imports nothing from the library.

The SANA-WM pages (paper analysis, abstract and method components) describe
the layer as frame-wise Gated DeltaNet: the SANA-Video linear attention whose
recurrent state gets decay gates and delta-rule corrections, keys scaled by
1/sqrt(D S).  They print no formula.  The reading fixed here keeps everything
of the base layer (ReLU feature map, the d x (d+1) state with its normaliser
column, queries of frame f reading S_f) and makes the frame's write a delta
rule: the frame's keys first read what the decayed state already holds for
them and write only the difference, scaled by a per-frame strength beta:

  a_f = sigmoid(g[f]),  beta_f = sigmoid(b[f]),  K~ = relu(K_f),  V1 = [V_f | 1]
  S_f = a_f S_{f-1} + beta_f K~^T (V1 - a_f K~ S_{f-1})
      = a_f (I - beta_f K~^T K~) S_{f-1} + beta_f K~^T V1
  out_t = relu(q_t) S_f[:, :d] / (relu(q_t) S_f[:, d] + eps)

With beta = 0 the state only decays; from a zero state the first frame's
output is the base layer's up to eps; with orthonormal key rows and
beta = a = 1 the frame's keys read back exactly its values (the delta rule's
defining property).  The pins are in tests/test_gdn_oracle.py.
"""

from __future__ import annotations

import numpy as np

__all__ = ["gla_gdn_head", "gla_gdn_forward"]


def _f64(x):
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def gla_gdn_head(q, k, v, g, beta_logits, T, state_in=None, eps=1e-6):
    """One (batch, head) slice: q, k, v [F*T, d], g and beta_logits [F];
    returns (out [F*T, d], state_out [d, d+1])."""
    q, k, v, g, bl = (_f64(x) for x in (q, k, v, g, beta_logits))
    g = g.reshape(-1)
    bl = bl.reshape(-1)
    F = g.shape[0]
    d = q.shape[1]
    S = np.zeros((d, d + 1)) if state_in is None else _f64(state_in).copy()
    out = np.zeros((F * T, d))
    for f in range(F):
        rows = slice(f * T, (f + 1) * T)
        a = _sigmoid(g[f])
        beta = _sigmoid(bl[f])
        Kf = np.maximum(k[rows], 0.0)
        V1 = np.hstack([v[rows], np.ones((T, 1))])
        # what the frame's keys read from the decayed state, then the delta write
        retrieved = Kf @ (a * S)
        S = a * S + beta * (Kf.T @ (V1 - retrieved))
        Qf = np.maximum(q[rows], 0.0)
        out[rows] = (Qf @ S[:, :d]) / (Qf @ S[:, d] + eps)[:, None]
    return out, S


def gla_gdn_forward(q, k, v, gate, beta_logits, frames, state_in=None, eps=1e-6):
    """Whole batch: q, k, v [B, F*T, H, d], gate and beta_logits [B, F, H],
    state [B, H, d, d+1]."""
    q, k, v, gate, bl = (_f64(x) for x in (q, k, v, gate, beta_logits))
    B, N, H, d = q.shape
    T = N // frames if frames else 0
    out = np.zeros_like(q)
    s_out = np.zeros((B, H, d, d + 1))
    s_in = None if state_in is None else _f64(state_in)
    for b in range(B):
        for h in range(H):
            o, s = gla_gdn_head(q[b, :, h], k[b, :, h], v[b, :, h], gate[b, :, h], bl[b, :, h], T,
                                None if s_in is None else s_in[b, h], eps)
            out[b, :, h] = o
            s_out[b, h] = s
    return out, s_out
