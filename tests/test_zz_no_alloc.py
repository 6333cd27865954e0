"""gla_forward_noalloc: the entry point for callers that must not allocate
device memory while they run the layer (for example a serving process whose
own allocator has reserved all free HBM, or a per-frame streaming loop that
must not enter the CUDA allocator).  It keeps its workspace in a fixed device
array inside the library.

Checked through the C ABI, on two or more calls in a row:
  * against the fp64 oracle, element by element, at the parity tests'
    tolerance (max|err| <= 1e-2 max|oracle|, rel-L2 <= 5e-3) on out and on
    the carried state;
  * against gla_forward bit for bit: both run the same kernels on the same
    tile schedule, only the workspace address differs, so any difference is a
    fault of the fixed array (a stale read, an overlap of its regions);
  * a larger problem first, then smaller ones at every head dim, so that the
    smaller calls run over what the larger one left in the array;
  * device memory use does not grow, and a problem that needs more than the
    fixed array is rejected before launch.
This file is collected last on purpose: it must also pass after every other
test has used the library in the same process.
"""

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, make_inputs, make_state

pytestmark = pytest.mark.gpu

TOL_MAX = 1e-2
TOL_L2 = 5e-3


def _close(gpu, ref, what):
    gpu = gpu.double().cpu().numpy() if hasattr(gpu, "cpu") else np.asarray(gpu, np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, what
    assert np.all(np.isfinite(gpu)), what
    err = np.abs(gpu - ref).max()
    assert err <= TOL_MAX * np.abs(ref).max(), "%s: max err %.3e" % (what, err)
    l2 = np.linalg.norm(gpu - ref) / np.linalg.norm(ref)
    assert l2 <= TOL_L2, "%s: rel L2 %.3e" % (what, l2)


@pytest.fixture(scope="module")
def gla():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gated_linear_attention_frame_b200.build import build

    build()
    import gated_linear_attention_frame_b200 as g

    g.load_library()
    return g


def _run(fn, w, q, k, v, g, state, out):
    """One call of `fn` (gla_forward or gla_forward_noalloc); `state` (device
    fp32) is updated in place."""
    fn(q, k, v, g, state, state, out, w.B, w.H, w.frames, w.tokens_per_frame, w.d, w.eps)


def _carried_calls(gla, w, calls, s0):
    """`calls` consecutive calls through both entry points, state carried;
    every output and the final state compared bitwise and with the oracle."""
    dev = torch.device("cuda")
    inputs = [make_inputs(w, call=c) for c in range(calls)]
    state_a = None if s0 is None else s0.to(dev).clone()
    state_b = None if s0 is None else s0.to(dev).clone()
    if state_a is None:
        state_a = torch.zeros(w.B, w.H, w.d, w.d + 1, device=dev)
        state_b = torch.zeros(w.B, w.H, w.d, w.d + 1, device=dev)
    ref_state = None if s0 is None else s0.double().numpy()
    for c, (q, k, v, g) in enumerate(inputs):
        qd, kd, vd, gd = (x.to(dev) for x in (q, k, v, g))
        out_a = torch.empty_like(qd)
        out_b = torch.empty_like(qd)
        _run(gla.gla_forward, w, qd, kd, vd, gd, state_a, out_a)
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        _run(gla.gla_forward_noalloc, w, qd, kd, vd, gd, state_b, out_b)
        torch.cuda.synchronize()
        free1 = torch.cuda.mem_get_info()[0]
        assert free1 >= free0, "gla_forward_noalloc took device memory (%d -> %d)" % (free0,
                                                                                      free1)
        ref_out, ref_state = oracle.gla_forward(q, k, v, g, w.frames, ref_state, w.eps)
        tag = "%s d=%d call %d" % (w.name, w.d, c)
        assert torch.equal(out_b, out_a), tag + ": out differs from gla_forward"
        assert torch.equal(state_b, state_a), tag + ": state differs from gla_forward"
        _close(out_b, ref_out, tag + " out")
    _close(state_b, ref_state, "%s d=%d state after %d calls" % (w.name, w.d, calls))
    assert gla.gla_device_fault() == 0


def test_noalloc_stream_step_two_calls(gla):
    # the one-frame streaming step: 8 sequences x 24 heads x 3680 tokens, d = 128,
    # random fp32 state carried from the first call into the second
    w = WORKLOADS["stream"]
    _carried_calls(gla, w, 2, make_state(w))


# Larger first, then smaller: the later calls run over what the earlier ones
# left in the shared array.  Several frames with ragged tails (T not a
# multiple of the 128-token tile), units split over CTAs, every head dim.
SHAPES = [
    # name, B, H, d, frames, T, random state_in
    ("multi-frame ragged", 2, 8, 128, 6, 300, False),   # 96 units, ~19 MB of scratch
    ("one head d=64", 1, 3, 64, 5, 131, True),
    ("two heads d=32", 2, 2, 32, 4, 77, True),
    ("tile split d=128", 1, 37, 128, 2, 400, True),
]


@pytest.mark.parametrize("name,B,H,d,F,T,state", SHAPES)
def test_noalloc_after_larger_calls(gla, name, B, H, d, F, T, state):
    w = WORKLOADS["tiny"].with_(name=name, B=B, H=H, d=d, frames=F, tokens_per_frame=T,
                                random_state_in=state)
    _carried_calls(gla, w, 2, make_state(w))


def test_noalloc_rejects_problems_beyond_its_scratch(gla):
    w = WORKLOADS["720p-5s"]  # needs ~110 MB of workspace
    dev = torch.device("cuda")
    q = torch.zeros(16, device=dev, dtype=torch.bfloat16)  # never read: rejected first
    g = torch.zeros(4, device=dev)
    with pytest.raises(gla.GLAError) as ei:
        gla.gla_forward_noalloc(q.data_ptr(), q.data_ptr(), q.data_ptr(), g.data_ptr(), None,
                                None, q.data_ptr(), w.B, w.H, w.frames, w.tokens_per_frame, w.d,
                                w.eps)
    assert ei.value.status == gla.GLA_ERR_SCRATCH
    assert gla.gla_noalloc_scratch_bytes() == 32 << 20
