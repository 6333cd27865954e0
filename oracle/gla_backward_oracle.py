"""fp64 CPU oracle for the gradients of block-causal gated linear attention.

TEST INFRASTRUCTURE ONLY (like gla_oracle.py): used by the tests and the
benchmark's CPU leg, never by the library; imports nothing from the library.

The layer (one (batch, head) slice; frames f, tokens t of frame f):
  q~ = relu(q), k~ = relu(k), a_f = sigmoid(g_f)
  S_f = a_f S_{f-1} + k~_f^T [v_f | 1]          (S_{-1} = state_in)
  num_t = q~_t S_f[:, :d], den_t = q~_t S_f[:, d] + eps, out_t = num_t / den_t
  state_out = S_{F-1}
Given dout (same shape as out) and dstate_out (same shape as the state, or
zero), the gradients of sum(dout * out) + sum(dstate_out * state_out) with
respect to q, k, v, g and state_in.

Two independent computations are provided:
  * gla_backward_head: the forward recurrence written in float64 torch ops
    and differentiated by torch.autograd (a library primitive serving as the
    step "differentiate");
  * gla_backward_head_manual: the chain rule written out step by step (the
    reverse recurrence G_f = dS_f + a_{f+1} G_{f+1}).
Both are pinned by central finite differences on tiny inputs
(tests/test_backward_oracle.py).

The pages (SANA-Video 2.0; the SANA-Video ICLR 2026 talk; SANA-WM) train the
model from scratch but print no gradient formula: the gradients are those of
the forward definition, nothing more.
"""

from __future__ import annotations

import numpy as np
import torch

__all__ = ["gla_forward_torch_head", "gla_backward_head", "gla_backward_head_manual",
           "gla_backward"]


def _t64(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64)
    return torch.as_tensor(np.asarray(x, dtype=np.float64))


def gla_forward_torch_head(q, k, v, g, T, state_in=None, eps=1e-6):
    """The forward recurrence in float64 torch ops (differentiable).
    q, k, v: [F*T, d]; g: [F]; state_in: [d, d+1] or None."""
    F = g.shape[0]
    d = q.shape[1]
    S = torch.zeros(d, d + 1, dtype=torch.float64) if state_in is None else state_in
    a = 1.0 / (1.0 + torch.exp(-g))
    ones = torch.ones(T, 1, dtype=torch.float64)
    outs = []
    for f in range(F):
        rows = slice(f * T, (f + 1) * T)
        Kf = torch.relu(k[rows])
        S = a[f] * S + Kf.T @ torch.cat([v[rows], ones], dim=1)
        Qf = torch.relu(q[rows])
        num = Qf @ S[:, :d]
        den = Qf @ S[:, d] + eps
        outs.append(num / den[:, None])
    out = torch.cat(outs, dim=0) if outs else torch.zeros(0, d, dtype=torch.float64)
    return out, S


def gla_backward_head(q, k, v, g, T, dout, state_in=None, dstate_out=None, eps=1e-6):
    """Gradients (dq, dk, dv, dg, dstate_in) of one (batch, head) slice by
    autograd of gla_forward_torch_head.  dstate_in is None when state_in is
    None (the zero state is not an input)."""
    q, k, v, g, dout = (_t64(x) for x in (q, k, v, g, dout))
    g = g.reshape(-1)
    leaves = [q.requires_grad_(), k.requires_grad_(), v.requires_grad_(), g.requires_grad_()]
    s_in = None
    if state_in is not None:
        s_in = _t64(state_in).requires_grad_()
        leaves.append(s_in)
    out, s_out = gla_forward_torch_head(q, k, v, g, T, s_in, eps)
    loss = (out * dout).sum()
    if dstate_out is not None:
        loss = loss + (s_out * _t64(dstate_out)).sum()
    grads = torch.autograd.grad(loss, leaves, allow_unused=True)
    grads = [torch.zeros_like(x) if gr is None else gr for gr, x in zip(grads, leaves)]
    dq, dk, dv, dg = (gr.numpy() for gr in grads[:4])
    ds_in = grads[4].numpy() if state_in is not None else None
    return dq, dk, dv, dg, ds_in


def gla_backward_head_manual(q, k, v, g, T, dout, state_in=None, dstate_out=None, eps=1e-6,
                             return_g=False):
    """The same gradients by the chain rule written out (numpy float64):
      dnum_t = dout_t / den_t,  dden_t = -(dout_t . out_t) / den_t
      dq_t   = 1[q_t > 0] * ([dnum_t | dden_t] S_f^T)
      dS_f   = sum_{t in f} q~_t^T [dnum_t | dden_t]
      G_f    = dS_f + a_{f+1} G_{f+1},   G_F = dstate_out
      da_f   = <G_f, S_{f-1}>,  dg_f = da_f a_f (1 - a_f),  dstate_in = a_0 G_0
      dk_t   = 1[k_t > 0] * ([v_t | 1] G_f^T),  dv_t = k~_t G_f[:, :d]
    With return_g, also returns the list of G_f (frame order) as a sixth item.
    """
    q, k, v, g, dout = (_t64(x).numpy() for x in (q, k, v, g, dout))
    g = g.reshape(-1)
    F = g.shape[0]
    d = q.shape[1]
    a = 1.0 / (1.0 + np.exp(-g))
    S_prev = np.zeros((d, d + 1)) if state_in is None else _t64(state_in).numpy().copy()
    states_before = []  # S_{f-1}
    states = []         # S_f
    for f in range(F):
        rows = slice(f * T, (f + 1) * T)
        states_before.append(S_prev)
        Kf = np.maximum(k[rows], 0.0)
        S = a[f] * S_prev + Kf.T @ np.hstack([v[rows], np.ones((T, 1))])
        states.append(S)
        S_prev = S
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dg = np.zeros(F)
    Gs = [None] * F
    G_next = np.zeros((d, d + 1)) if dstate_out is None else _t64(dstate_out).numpy().copy()
    a_next = 1.0
    for f in range(F - 1, -1, -1):
        rows = slice(f * T, (f + 1) * T)
        S = states[f]
        Qf = np.maximum(q[rows], 0.0)
        num = Qf @ S[:, :d]
        den = Qf @ S[:, d] + eps
        out = num / den[:, None]
        dnum = dout[rows] / den[:, None]
        dden = -np.sum(dout[rows] * out, axis=1) / den
        Dm = np.hstack([dnum, dden[:, None]])           # [T, d+1]
        dq[rows] = (q[rows] > 0) * (Dm @ S.T)
        dS = Qf.T @ Dm                                  # [d, d+1]
        G = dS + a_next * G_next if f < F - 1 else dS + G_next
        da = float(np.sum(G * states_before[f]))
        dg[f] = da * a[f] * (1.0 - a[f])
        Kf = np.maximum(k[rows], 0.0)
        V1 = np.hstack([v[rows], np.ones((T, 1))])
        dk[rows] = (k[rows] > 0) * (V1 @ G.T)
        dv[rows] = Kf @ G[:, :d]
        Gs[f] = G
        G_next = G
        a_next = a[f]
    ds_in = None
    if state_in is not None:
        ds_in = a[0] * G_next if F > 0 else G_next
    if return_g:
        return dq, dk, dv, dg, ds_in, Gs
    return dq, dk, dv, dg, ds_in


def gla_backward(q, k, v, gate_logits, frames, dout, state_in=None, dstate_out=None, eps=1e-6):
    """Whole batch ([B, F*T, H, d] tensors, gate [B, F, H], state [B, H, d, d+1])
    by gla_backward_head_manual on every (b, h)."""
    q, k, v, dout = (_t64(x).numpy() for x in (q, k, v, dout))
    g = _t64(gate_logits).numpy()
    B, N, H, d = q.shape
    T = N // frames if frames else 0
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dg = np.zeros((B, frames, H))
    ds = None if state_in is None else np.zeros((B, H, d, d + 1))
    s_in = None if state_in is None else _t64(state_in).numpy()
    ds_out = None if dstate_out is None else _t64(dstate_out).numpy()
    for b in range(B):
        for h in range(H):
            r = gla_backward_head_manual(q[b, :, h], k[b, :, h], v[b, :, h], g[b, :, h], T,
                                         dout[b, :, h], None if s_in is None else s_in[b, h],
                                         None if ds_out is None else ds_out[b, h], eps)
            dq[b, :, h], dk[b, :, h], dv[b, :, h], dg[b, :, h] = r[:4]
            if ds is not None:
                ds[b, h] = r[4]
    return dq, dk, dv, dg, ds
