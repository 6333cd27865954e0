"""Parity of gla_softmax_anchor (through the C ABI) with the fp64 oracle.

Tolerance as the linear layers: max|gpu - oracle| <= 1e-2 max|oracle| and
rel-L2 <= 5e-3.  Small shapes cover ragged key and query tiles, sinks shorter
than, equal to and longer than a frame, windows of 1 to all frames, the
output gate, several units per CTA; the 720p-5s shape runs at full size (a
window of 2 frames, the first frame as sinks, the output gate: the benchmark's
launch) and is compared on sampled (batch, head) slices.
"""

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, anchor_workload, make_anchor_gate, make_inputs

pytestmark = pytest.mark.gpu

TOL_MAX = 1e-2
TOL_L2 = 5e-3


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gated_linear_attention_frame_b200.build import build

    build()
    import gated_linear_attention_frame_b200 as g

    g.load_library()
    yield g
    assert g.gla_device_fault() == 0


def assert_close(gpu, ref, what=""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, what
    assert np.all(np.isfinite(gpu)), what + ": non-finite values"
    err = np.abs(gpu - ref)
    scale = np.abs(ref).max()
    l2 = np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-300)
    assert err.max() <= TOL_MAX * scale, "%s: max err %.3e > %.1e * %.3e" % (what, err.max(),
                                                                            TOL_MAX, scale)
    assert l2 <= TOL_L2, "%s: rel L2 %.3e > %.1e" % (what, l2, TOL_L2)


def case(B, H, F, T, seed, gate):
    w = WORKLOADS["tiny"].with_(B=B, H=H, frames=F, tokens_per_frame=T, d=128, k_scaled=False)
    q, k, v, _ = make_inputs(w, seed=seed)
    z = None
    if gate:
        z = (torch.randn(q.shape, generator=torch.Generator().manual_seed(seed + 5))
             .to(torch.bfloat16))
    return q, k, v, z


def run_gpu(q, k, v, z, F, W, S):
    import gated_linear_attention_frame_b200 as gla

    dev = torch.device("cuda")
    out = gla.softmax_anchor(q.to(dev), k.to(dev), v.to(dev), F, W, S,
                             None if z is None else z.to(dev))
    torch.cuda.synchronize()
    return out.float().cpu().numpy()


SMALL = [
    # B, H, F, T, window, n_sink, gate
    (1, 2, 3, 200, 2, 0, False),
    (1, 2, 4, 130, 2, 130, True),    # sinks = the first frame
    (2, 1, 5, 64, 1, 20, False),     # frame-local + a few sinks
    (1, 3, 4, 100, 4, 0, True),      # window = every frame: block-causal
    (1, 1, 6, 50, 2, 120, False),    # sinks longer than two frames
    (1, 2, 1, 300, 1, 0, False),     # one frame: full attention
    (2, 37, 2, 128, 2, 64, True),    # more units than CTAs
    (1, 1, 3, 1, 2, 1, False),       # one token per frame
]


@pytest.mark.parametrize("B,H,F,T,W,S,gate", SMALL)
def test_small_shapes_full_compare(B, H, F, T, W, S, gate):
    q, k, v, z = case(B, H, F, T, 8000 + B * 100 + H * 10 + F + T, gate)
    out = run_gpu(q, k, v, z, F, W, S)
    ref = oracle.softmax_anchor_forward(q, k, v, F, W, S, z)
    assert_close(out, ref, "out")


def test_full_size_720p_5s_sampled_heads():
    import gated_linear_attention_frame_b200 as gla

    w = anchor_workload(WORKLOADS["720p-5s"])
    dev = torch.device("cuda")
    q, k, v, _ = make_inputs(w, device=dev)
    z = make_anchor_gate(w, device=dev)
    T = w.tokens_per_frame
    out = gla.softmax_anchor(q, k, v, w.frames, 2, T, z)
    torch.cuda.synchronize()
    for b, h in [(0, 0), (1, 17)]:
        sl = lambda x: x[b, :, h].float().cpu().numpy()  # noqa: E731
        ref = oracle.softmax_anchor_head(sl(q), sl(k), sl(v), T, 2, T, sl(z))
        assert_close(sl(out), ref, "out[b=%d,h=%d]" % (b, h))


@pytest.mark.parametrize("gate", [False, True])
def test_growing_scores_rescale_the_accumulator(gate):
    """Keys of frame f scaled by 1 + 4 f: with a window over every frame each
    new frame raises the row maxima far beyond the kernel's rescale threshold,
    so the running accumulator is rescaled many times per query tile."""
    B, H, F, T = 1, 2, 4, 200
    q, k, v, z = case(B, H, F, T, 8100, gate)
    scale = torch.repeat_interleave(1.0 + 4.0 * torch.arange(F, dtype=torch.float32), T)
    k = (k.float() * scale[None, :, None, None]).to(torch.bfloat16)
    out = run_gpu(q, k, v, z, F, F, 0)
    ref = oracle.softmax_anchor_forward(q, k, v, F, F, 0, z)
    assert_close(out, ref, "out")
