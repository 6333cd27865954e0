"""fp64 CPU oracle of gated linear attention with 3D rotary position embedding.

TEST INFRASTRUCTURE ONLY (like gla_oracle.py): used by the tests and the
benchmark's CPU legs, never by the library; imports nothing from the library.

The SANA-Video ICLR 2026 talk (temporal modelling segment) adds a 3D RoPE to
the linear attention and gives no formula.  The reading fixed here (linear
attention with rotary embedding in the RoFormer form: rotate the feature-mapped
query and key in the numerator only, keep the normaliser on the un-rotated
features so that it stays positive):

  position of token t of frame f:  (p_t, p_y, p_x) = (frame_offset + f, t // grid_w, t % grid_w)
  head dim d = d_t + d_y + d_x (each a multiple of 8), features laid out
      [temporal | height | width]; pair j of an axis block with n features
      rotates features (2j, 2j+1) of the block by the angle p_axis * theta^(-2j/n)
  R_t = the block-diagonal rotation of token t; q^_t = R_t phi(q_t), k^_t = R_t phi(k_t)
  S_f[:, :d] = a_f S_{f-1}[:, :d] + K^_f^T V_f
  S_f[:, d]  = a_f S_{f-1}[:, d]  + phi(K_f)^T 1
  out_t      = q^_t S_f[:, :d] / (phi(q_t) S_f[:, d] + eps)

With every angle zero (d_t = d, frame_offset = 0, one frame) it is the layer
of gla_oracle.gla_head.  The pins are in tests/test_rope_oracle.py.
"""

from __future__ import annotations

import numpy as np

__all__ = ["rope_pair_angles", "rope_rotate", "gla_rope_head", "gla_rope_forward",
           "gla_rope_bruteforce_head"]


def _f64(x):
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def rope_pair_angles(pos_t, pos_y, pos_x, dims, theta):
    """Angles [n_tokens, d/2] of the d/2 feature pairs, for tokens at the
    given integer positions (1-D arrays of equal length)."""
    d_t, d_y, d_x = dims
    cols = []
    for pos, n in ((pos_t, d_t), (pos_y, d_y), (pos_x, d_x)):
        j = np.arange(n // 2, dtype=np.float64)
        freq = theta ** (-2.0 * j / n) if n else np.zeros(0)
        cols.append(np.outer(np.asarray(pos, dtype=np.float64), freq))
    return np.concatenate(cols, axis=1)


def rope_rotate(x, angles):
    """Rotate pairs (x[:, 2j], x[:, 2j+1]) by angles[:, j] (counter-clockwise)."""
    c, s = np.cos(angles), np.sin(angles)
    x0, x1 = x[:, 0::2], x[:, 1::2]
    y = np.empty_like(x)
    y[:, 0::2] = x0 * c - x1 * s
    y[:, 1::2] = x0 * s + x1 * c
    return y


def _frame_angles(T, f, frame_offset, grid_w, dims, theta):
    t = np.arange(T)
    return rope_pair_angles(np.full(T, frame_offset + f), t // grid_w, t % grid_w, dims, theta)


def gla_rope_head(q, k, v, g, T, grid_w, frame_offset=0, dims=None, theta=10000.0,
                  state_in=None, eps=1e-6):
    """One (batch, head) slice: q, k, v [F*T, d], g [F]; returns (out, state_out)."""
    q, k, v, g = (_f64(x) for x in (q, k, v, g))
    g = g.reshape(-1)
    F = g.shape[0]
    d = q.shape[1]
    dims = tuple(dims) if dims is not None else (d, 0, 0)
    assert sum(dims) == d and all(n % 8 == 0 for n in dims)
    S = np.zeros((d, d + 1)) if state_in is None else _f64(state_in).copy()
    out = np.zeros((F * T, d))
    for f in range(F):
        rows = slice(f * T, (f + 1) * T)
        a = 1.0 / (1.0 + np.exp(-g[f]))
        ang = _frame_angles(T, f, frame_offset, grid_w, dims, theta)
        Kf = np.maximum(k[rows], 0.0)
        S[:, :d] = a * S[:, :d] + rope_rotate(Kf, ang).T @ v[rows]
        S[:, d] = a * S[:, d] + Kf.sum(axis=0)
        Qf = np.maximum(q[rows], 0.0)
        out[rows] = (rope_rotate(Qf, ang) @ S[:, :d]) / (Qf @ S[:, d] + eps)[:, None]
    return out, S


def gla_rope_forward(q, k, v, gate, frames, grid_w, frame_offset=0, dims=None, theta=10000.0,
                     state_in=None, eps=1e-6):
    """Whole batch: q, k, v [B, F*T, H, d], gate [B, F, H], state [B, H, d, d+1]."""
    q, k, v, gate = (_f64(x) for x in (q, k, v, gate))
    B, N, H, d = q.shape
    T = N // frames if frames else 0
    out = np.zeros_like(q)
    s_out = np.zeros((B, H, d, d + 1))
    s_in = None if state_in is None else _f64(state_in)
    for b in range(B):
        for h in range(H):
            o, s = gla_rope_head(q[b, :, h], k[b, :, h], v[b, :, h], gate[b, :, h], T, grid_w,
                                 frame_offset, dims, theta, None if s_in is None else s_in[b, h],
                                 eps)
            out[b, :, h] = o
            s_out[b, h] = s
    return out, s_out


def gla_rope_bruteforce_head(q, k, v, g, T, grid_w, frame_offset=0, dims=None, theta=10000.0,
                             eps=1e-6):
    """Quadratic form with zero initial state, the rotation written in
    complex numbers: pair j of a feature vector is z = x_{2j} + i x_{2j+1};
    rotating by an angle multiplies z by exp(i angle), so
        (R_i u) . (R_j w) = Re sum_pairs conj(u) w exp(i (angle_j - angle_i)).
    out_i = sum_{j: f(j) <= f(i)} (prod_{m=f(j)+1}^{f(i)} a_m) Re(...) v_j
            / (sum_j (same product) phi(q_i) . phi(k_j) + eps)."""
    q, k, v, g = (_f64(x) for x in (q, k, v, g))
    g = g.reshape(-1)
    F = g.shape[0]
    d = q.shape[1]
    dims = tuple(dims) if dims is not None else (d, 0, 0)
    a = 1.0 / (1.0 + np.exp(-g))
    n = F * T
    frame = np.arange(n) // T
    t = np.arange(n) % T
    pos = (frame_offset + frame, t // grid_w, t % grid_w)
    ang = rope_pair_angles(*pos, dims, theta)           # [n, d/2]
    Q = np.maximum(q, 0.0)
    K = np.maximum(k, 0.0)
    zq = Q[:, 0::2] + 1j * Q[:, 1::2]
    zk = K[:, 0::2] + 1j * K[:, 1::2]
    out = np.zeros((n, d))
    for i in range(n):
        num = np.zeros(d)
        den = 0.0
        for j in range(n):
            if frame[j] > frame[i]:
                continue
            w = 1.0
            for m in range(frame[j] + 1, frame[i] + 1):  # the key's own frame adds undecayed
                w *= a[m]
            rot = np.real(np.sum(np.conj(zq[i]) * zk[j] * np.exp(1j * (ang[j] - ang[i]))))
            num += w * rot * v[j]
            den += w * float(Q[i] @ K[j])
        out[i] = num / (den + eps)
    return out
