"""fp64 CPU oracle for block-causal gated linear attention (one frame per chunk).

TEST INFRASTRUCTURE ONLY.  This module is the slow, plain reference that the
CUDA library is checked against.  Only the test suite, the package's smoke
check and the benchmark's CPU-baseline leg may import it; the library never
does, and this module imports nothing from the library.

What it computes
----------------
The pages describe the structure of the linear-attention layer but print no
formulas:

* SANA-Video 2.0 (project page, "Hybrid Linear-Softmax Attention"; the
  abstract on the author page): gated linear attention is the O(N) token
  mixer of the hybrid DiT.
* SANA-Video ICLR 2026 oral talk (block KV cache / block-causal linear
  attention segment): the linear-attention state is a fixed-size D x D
  matrix; block i adds its own key-value contribution to the state cached
  after block i-1, and the block's queries read the updated state.  Memory is
  constant in the sequence length.
* SANA-WM paper analysis (method components): plain cumulative linear
  attention has no decay and drifts over long sequences; decay gates on the
  recurrent state fix that; the attention is applied frame-wise.

The layer definition used here fixes the open parts as follows:
  phi(x)  = max(x, 0)                               (feature map)
  a_f     = 1 / (1 + exp(-g[f]))                    (per frame, per head)
  S_f     = a_f * S_{f-1} + phi(K_f)^T [V_f | 1]    (d x (d+1); S_{-1} = state_in)
  out_t   = (phi(q_t) S_f[:, :d]) / (phi(q_t) S_f[:, d] + eps)   for t in frame f
  state_out = S_{F-1}
Queries of frame f read S_f, so attention is bidirectional inside a frame and
causal across frames.  Every step is written out literally, in float64.

Parity status: pinned (tests/test_oracle.py) by a brute-force quadratic form,
closed forms (a = 1 one frame, a = 0, a = 1 many frames), a hand-worked
example (tests/golden/), streaming/chunking invariance and invariants.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "sigmoid",
    "relu",
    "gla_head",
    "gla_forward",
    "gla_bruteforce_head",
]


def _f64(x):
    """Widen any array-like (numpy, or torch CPU tensor incl. bf16) to float64."""
    if hasattr(x, "detach"):  # torch tensor: widen through fp32 (exact for bf16)
        x = x.detach().to("cpu").float().numpy()
    return np.asarray(x, dtype=np.float64)


def sigmoid(g):
    """Decay a = 1/(1+exp(-g)) in float64 (g = +inf -> 1, g = -inf -> 0)."""
    g = _f64(g)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-g))


def relu(x):
    """Feature map phi(x) = max(x, 0); maps -0 to +0."""
    return np.maximum(_f64(x), 0.0) + 0.0


def gla_head(q, k, v, g, T, state_in=None, eps=1e-6):
    """One (batch, head) slice: the per-frame recurrence, frame by frame.

    q, k, v : [F*T, d]  (any real dtype; widened to float64)
    g       : [F]       gate logits of this head
    state_in: [d, d+1]  or None for the zero state
    Returns (out [F*T, d] float64, state_out [d, d+1] float64).

    Follows the block KV-cache description of the SANA-Video talk: for each
    block (here: one latent frame) the block's contribution phi(K)^T [V | 1]
    is added to the cached state after the cache is scaled by the frame's
    decay, and the block's queries then read the updated state.
    """
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(g).reshape(-1)
    F = g.shape[0]
    d = q.shape[1]
    if q.shape[0] != F * T:
        raise ValueError("q has %d rows, expected frames*T = %d" % (q.shape[0], F * T))
    S = np.zeros((d, d + 1)) if state_in is None else _f64(state_in).copy()
    out = np.zeros((F * T, d))
    a = sigmoid(g)
    ones = np.ones((T, 1))
    for f in range(F):
        rows = slice(f * T, (f + 1) * T)
        Kf = relu(k[rows])                      # phi(K_f)      [T, d]
        Vf1 = np.hstack([v[rows], ones])        # [V_f | 1]     [T, d+1]
        S = a[f] * S + Kf.T @ Vf1               # decay the carried state, add the frame
        Qf = relu(q[rows])                      # phi(Q_f)      [T, d]
        num = Qf @ S[:, :d]                     # [T, d]
        den = Qf @ S[:, d]                      # [T]
        out[rows] = num / (den + eps)[:, None]
    return out, S


def gla_forward(q, k, v, gate_logits, frames, state_in=None, eps=1e-6):
    """Whole batch: q, k, v [B, F*T, H, d]; gate_logits [B, F, H];
    state_in [B, H, d, d+1] or None.  Returns (out [B, F*T, H, d],
    state_out [B, H, d, d+1]), both float64.  Heads and batch entries are
    independent, so this is gla_head on every (b, h)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    g = _f64(gate_logits)
    B, N, H, d = q.shape
    F = int(frames)
    if F == 0:
        if N != 0:
            raise ValueError("frames = 0 requires an empty token axis")
        T = 0
    else:
        if N % F:
            raise ValueError("token axis %d is not a multiple of frames %d" % (N, F))
        T = N // F
    out = np.zeros((B, N, H, d))
    s_out = np.zeros((B, H, d, d + 1))
    s_in = None if state_in is None else _f64(state_in)
    for b in range(B):
        for h in range(H):
            o, s = gla_head(q[b, :, h], k[b, :, h], v[b, :, h], g[b, :, h], T,
                            None if s_in is None else s_in[b, h], eps)
            out[b, :, h] = o
            s_out[b, h] = s
    return out, s_out


def gla_bruteforce_head(q, k, v, g, T, state_in=None, eps=1e-6):
    """Quadratic (attention-matrix) form of the same layer for one head.

    Written from the definition by unrolling the recurrence, with frames
    counted from 0 and f(j) the frame of token j:
      S_f = (prod_{m=0}^{f} a_m) S_in + sum_{f' <= f} (prod_{m=f'+1}^{f} a_m) dS_{f'}
    so for a query i in frame f(i)
      num_i = sum_{j: f(j) <= f(i)} w(j, i) (phi(q_i).phi(k_j)) v_j + P_i phi(q_i)^T S_in[:, :d]
      den_i = sum_{j: f(j) <= f(i)} w(j, i) (phi(q_i).phi(k_j))     + P_i phi(q_i)^T S_in[:, d]
      out_i = num_i / (den_i + eps)
    with w(j, i) = prod_{m=f(j)+1}^{f(i)} a_m and P_i = prod_{m=0}^{f(i)} a_m.
    Each weight is a product taken term by term, each pair (i, j) visited on
    its own: O(N^2 d), meant for tiny inputs only.
    """
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(g).reshape(-1)
    F = g.shape[0]
    N, d = q.shape
    a = sigmoid(g)
    fq = np.arange(N) // T if T > 0 else np.zeros(0, dtype=int)
    pq, pk = relu(q), relu(k)
    s_in = None if state_in is None else _f64(state_in)
    out = np.zeros((N, d))
    for i in range(N):
        fi = fq[i]
        num = np.zeros(d)
        den = 0.0
        for j in range(N):
            fj = fq[j]
            if fj > fi:
                continue
            w = 1.0
            for m in range(fj + 1, fi + 1):
                w *= a[m]
            s = float(pq[i] @ pk[j])
            num += w * s * v[j]
            den += w * s
        if s_in is not None:
            P = 1.0
            for m in range(0, fi + 1):
                P *= a[m]
            num += P * (pq[i] @ s_in[:, :d])
            den += P * float(pq[i] @ s_in[:, d])
        out[i] = num / (den + eps)
    # final state by the same unrolling (used to pin state_out)
    S = np.zeros((d, d + 1))
    for j in range(N):
        w = 1.0
        for m in range(fq[j] + 1, F):
            w *= a[m]
        S[:, :d] += w * np.outer(pk[j], v[j])
        S[:, d] += w * pk[j]
    if s_in is not None:
        P = 1.0
        for m in range(F):
            P *= a[m]
        S += P * s_in
    return out, S
