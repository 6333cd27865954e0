"""gla_softmax_anchor_step: the anchor layer one frame at a time, from the sink
and window caches, as a rollout runs it (through the C ABI).

Every frame of a sequence is run on its own, with its sink cache (the first
n_sink keys and values) and its window cache (the window's earlier frames,
oldest first) cut from the sequence, and compared
  * bit for bit with the same frame of one gla_softmax_anchor call over the
    whole sequence (the step reads the same key tiles in the same order), and
  * with the fp64 oracle over the whole sequence, at the parity tolerance
    (max|err| <= 1e-2 max|oracle|, rel-L2 <= 5e-3).
Shapes cover sinks shorter than, equal to and longer than a frame, windows of
one frame to all frames, ragged frames, the output gate, and the first frames
of a rollout (no sinks yet, a short window).
"""

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

TOL_MAX = 1e-2
TOL_L2 = 5e-3


@pytest.fixture(scope="module")
def gla():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gated_linear_attention_frame_b200.build import build

    build()
    import gated_linear_attention_frame_b200 as g

    g.load_library()
    yield g
    assert g.gla_device_fault() == 0


def _close(gpu, ref, what):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(gpu)), what
    err = np.abs(gpu - ref).max()
    assert err <= TOL_MAX * np.abs(ref).max(), "%s: max err %.3e" % (what, err)
    l2 = np.linalg.norm(gpu - ref) / np.linalg.norm(ref)
    assert l2 <= TOL_L2, "%s: rel L2 %.3e" % (what, l2)


CASES = [
    # B, H, F, T, window, n_sink, gate
    (1, 2, 4, 200, 2, 200, True),    # the first frame as sinks
    (2, 1, 5, 130, 3, 70, False),    # sinks shorter than a frame, ragged frames
    (1, 2, 4, 96, 2, 250, True),     # sinks longer than a frame
    (1, 1, 3, 64, 1, 0, False),      # frame-local attention only
    (1, 3, 3, 150, 3, 40, True),     # the window covers every frame
]


@pytest.mark.parametrize("B,H,F,T,W,n_sink,gate", CASES)
def test_rollout_steps_match_whole_sequence(gla, B, H, F, T, W, n_sink, gate):
    w = WORKLOADS["tiny"].with_(B=B, H=H, frames=F, tokens_per_frame=T, d=128, k_scaled=False)
    q, k, v, _ = make_inputs(w, seed=900 + F * 10 + T)
    z = None
    if gate:
        z = torch.randn(q.shape, generator=torch.Generator().manual_seed(7 + T)).to(torch.bfloat16)
    dev = torch.device("cuda")
    qd, kd, vd = (x.to(dev) for x in (q, k, v))
    zd = None if z is None else z.to(dev)
    whole = gla.softmax_anchor(qd, kd, vd, F, W, n_sink, zd)
    ref = oracle.softmax_anchor_forward(q, k, v, F, W, n_sink, z)
    sink_k = kd[:, :n_sink].contiguous() if n_sink > 0 else None
    sink_v = vd[:, :n_sink].contiguous() if n_sink > 0 else None
    for f in range(F):
        rows = slice(f * T, (f + 1) * T)
        lo = max(0, f - W + 1)
        win_k = kd[:, lo * T:f * T].contiguous() if f > lo else None
        win_v = vd[:, lo * T:f * T].contiguous() if f > lo else None
        out = gla.softmax_anchor_step(
            qd[:, rows].contiguous(), kd[:, rows].contiguous(), vd[:, rows].contiguous(), f, W,
            n_sink, sink_k, sink_v, win_k, win_v,
            None if zd is None else zd[:, rows].contiguous())
        torch.cuda.synchronize()
        assert torch.equal(out, whole[:, rows]), "frame %d differs from the whole-sequence call" % f
        _close(out.float().cpu().numpy(), ref[:, rows], "frame %d" % f)


def test_step_rejects_missing_caches(gla):
    dev = torch.device("cuda")
    x = torch.zeros(1, 64, 1, 128, dtype=torch.bfloat16, device=dev)
    # frame 3 with a window of 2 needs the window cache (frame 2) and the sinks
    with pytest.raises(gla.GLAError) as ei:
        gla.softmax_anchor_step(x, x, x, 3, 2, 64, x, x, None, None)
    assert ei.value.status == gla.GLA_ERR_NULL
    with pytest.raises(gla.GLAError) as ei:
        gla.softmax_anchor_step(x, x, x, 3, 2, 64, None, None, x, x)
    assert ei.value.status == gla.GLA_ERR_NULL
    # frame 0 needs neither
    gla.softmax_anchor_step(x, x, x, 0, 2, 64)
    torch.cuda.synchronize()
