"""Seeded synthetic inputs for the gated linear attention layer.

This module only draws random tensors with the shapes and distributions of
the layer workloads; it holds none of the layer's arithmetic.  Both the CUDA
library's tests/benchmark and the fp64 oracle receive exactly the tensors
produced here.

Shapes come from the SANA-Video 2.0 pages: 720p video is 736x1280 pixels
(Hugging Face Space page, "720p preview" profile), which a 16x spatial
compression turns into a 46x80 latent grid of 3680 tokens per latent frame;
480p gives 30x52 = 1560.  Five seconds at 16 FPS is 81 pixel frames, i.e. 21
latent frames after 4x temporal compression; one minute gives 241.  The
compression factors are not on the pages; the grid sizes are fixed by the
workload table below.

Layouts (all row-major, contiguous):
  q, k, v, out : bf16 [B, frames * tokens_per_frame, H, d], token n = f*T + t
  gate_logits  : fp32 [B, frames, H]
  state        : fp32 [B, H, d, d + 1]   (last column = normaliser)
"""

from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs", "make_state", "make_grads", "make_beta",
           "gdn_workload", "rope_dims", "seed_for", "anchor_workload", "make_anchor_gate"]

BASE_SEED = 20261202


@dataclass(frozen=True)
class Workload:
    name: str
    index: int          # position in the workload table (drives the seed)
    B: int
    H: int
    d: int
    frames: int
    tokens_per_frame: int
    g_mu: float         # gate logits ~ N(g_mu, g_sigma)
    g_sigma: float
    k_scaled: bool      # k drawn N(0,1) / sqrt(d) when True, else N(0,1)
    random_state_in: bool
    calls: int = 1      # consecutive streaming calls (state carried)
    eps: float = 1e-6
    grid_w: int = 1     # latent grid width (token t of a frame sits at row t // grid_w)
    k_div_tokens: bool = False  # k further divided by sqrt(tokens_per_frame) (delta-rule
                                # variant: the pages' 1/sqrt(D S) key scale)

    @property
    def tokens(self) -> int:
        """Tokens per sequence (frames * tokens_per_frame)."""
        return self.frames * self.tokens_per_frame

    @property
    def total_tokens(self) -> int:
        """Tokens per call over the whole batch (B * frames * T)."""
        return self.B * self.tokens

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS: dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny", 0, B=1, H=2, d=32, frames=4, tokens_per_frame=16,
                 g_mu=2.0, g_sigma=1.0, k_scaled=False, random_state_in=False, grid_w=4),
        Workload("480p-5s", 1, B=2, H=20, d=128, frames=21, tokens_per_frame=1560,
                 g_mu=3.0, g_sigma=1.0, k_scaled=True, random_state_in=False, grid_w=52),
        Workload("720p-5s", 2, B=2, H=24, d=128, frames=21, tokens_per_frame=3680,
                 g_mu=3.0, g_sigma=1.0, k_scaled=True, random_state_in=False, grid_w=80),
        Workload("720p-60s", 3, B=1, H=24, d=128, frames=241, tokens_per_frame=3680,
                 g_mu=4.0, g_sigma=0.5, k_scaled=True, random_state_in=False, grid_w=80),
        Workload("stream", 4, B=8, H=24, d=128, frames=1, tokens_per_frame=3680,
                 g_mu=3.0, g_sigma=1.0, k_scaled=False, random_state_in=True,
                 calls=64, grid_w=80),
    ]
}


def rope_dims(d: int) -> tuple[int, int, int]:
    """Feature blocks [temporal | height | width] of the rotary variant: a
    quarter of the head dim for time, the rest split between the two spatial
    axes (multiples of 8)."""
    return {32: (8, 8, 16), 64: (16, 24, 24), 128: (32, 48, 48)}[d]


def seed_for(w: Workload, call: int = 0) -> int:
    """Seed of call `call` of workload `w`: base + table index + 1000 * call."""
    return BASE_SEED + w.index + 1000 * call


def _normal(shape, gen, device):
    return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)


def make_inputs(w: Workload, call: int = 0, device="cpu", seed: int | None = None):
    """Draw (q, k, v, gate_logits) for one call of workload `w`.

    q, k, v are drawn in fp32 from N(0, 1) (k divided by sqrt(d) when the
    workload says so) and rounded to bf16 with round-to-nearest-even; gate
    logits are fp32 N(g_mu, g_sigma).  Tensors are drawn in the order q, k,
    v, g from one generator seeded with `seed_for(w, call)` (or `seed`).
    The same seed gives the same tensors on the same device type.
    """
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed_for(w, call) if seed is None else seed)
    shape = (w.B, w.tokens, w.H, w.d)
    q = _normal(shape, gen, dev).to(torch.bfloat16)
    k = _normal(shape, gen, dev)
    if w.k_scaled:
        k.mul_(1.0 / math.sqrt(w.d))
    if w.k_div_tokens and w.tokens_per_frame > 0:
        k.mul_(1.0 / math.sqrt(w.tokens_per_frame))
    k = k.to(torch.bfloat16)
    v = _normal(shape, gen, dev).to(torch.bfloat16)
    g = _normal((w.B, w.frames, w.H), gen, dev).mul_(w.g_sigma).add_(w.g_mu)
    return q, k, v, g


def make_state(w: Workload, device="cpu", seed: int | None = None):
    """Initial fp32 state [B, H, d, d+1]: N(0, 1) when the workload carries a
    random state, else None (zero state)."""
    if not w.random_state_in:
        return None
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed((seed_for(w) if seed is None else seed) + 7)
    return _normal((w.B, w.H, w.d, w.d + 1), gen, dev)


def make_grads(w: Workload, device="cpu", seed: int | None = None, dstate_out: bool = False,
               dstate_scale: float = 1e-3):
    """Upstream gradients for the backward pass: dout bf16 [B, tokens, H, d]
    ~ N(0, 1) rounded to nearest even, and (if `dstate_out`) an fp32
    [B, H, d, d+1] state gradient ~ N(0, dstate_scale^2), else None.  Drawn in
    that order from a generator seeded with seed_for(w) + 11 (or `seed`)."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed((seed_for(w) if seed is None else seed) + 11)
    dout = _normal((w.B, w.tokens, w.H, w.d), gen, dev).to(torch.bfloat16)
    ds = None
    if dstate_out:
        ds = _normal((w.B, w.H, w.d, w.d + 1), gen, dev).mul_(dstate_scale)
    return dout, ds


def gdn_workload(w: Workload) -> Workload:
    """The delta-rule variant of a workload: keys scaled by 1/sqrt(d T) (the
    SANA-WM pages' 1/sqrt(D S), S = tokens per frame), same shapes and seeds."""
    return w.with_(k_scaled=True, k_div_tokens=True)


def make_beta(w: Workload, device="cpu", seed: int | None = None):
    """Write-strength logits of the delta-rule variant: fp32 [B, frames, H]
    ~ N(0, 1), from a generator seeded with seed_for(w) + 13 (or `seed`)."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed((seed_for(w) if seed is None else seed) + 13)
    return _normal((w.B, w.frames, w.H), gen, dev)


def anchor_workload(w: Workload) -> Workload:
    """The softmax anchor layer's inputs for a workload: the same shapes and
    seeds with q, k ~ N(0, 1) unscaled, so that the scores q . k / sqrt(d) are
    ~ N(0, 1)."""
    return w.with_(k_scaled=False, k_div_tokens=False)


def make_anchor_gate(w: Workload, device="cpu", seed: int | None = None):
    """Output-gate logits z of the softmax anchor layer: bf16 [B, tokens, H, d]
    ~ N(0, 1) rounded to nearest even, from a generator seeded with
    seed_for(w) + 17 (or `seed`)."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed((seed_for(w) if seed is None else seed) + 17)
    return _normal((w.B, w.tokens, w.H, w.d), gen, dev).to(torch.bfloat16)
