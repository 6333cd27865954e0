"""gla_forward_noalloc: the entry point for callers that must not allocate
device memory while they run the layer (for example a serving process whose
own allocator has reserved all free HBM, or a per-frame streaming loop that
must not enter the CUDA allocator).  It keeps its workspace in a fixed device
array inside the library.

Checked through the C ABI against gla_forward on two calls in a row, with the
state of the first call carried into the second (the streaming use), within
the tolerance of the parity tests; device memory use must not grow, and a
problem that needs more than the fixed array is rejected before launch.
This file is collected last on purpose: it must also pass after every other
test has used the library in the same process.
"""

import numpy as np
import pytest
import torch

from workloads import WORKLOADS, make_inputs, make_state

pytestmark = pytest.mark.gpu

TOL_MAX = 1e-2
TOL_L2 = 5e-3


def _close(a, b, what):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    assert np.all(np.isfinite(a)), what
    err = np.abs(a - b).max()
    assert err <= TOL_MAX * np.abs(b).max(), "%s: max err %.3e" % (what, err)
    l2 = np.linalg.norm(a - b) / np.linalg.norm(b)
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


def test_noalloc_matches_forward_two_calls(gla):
    # the one-frame streaming step: 8 sequences x 24 heads x 3680 tokens, d = 128
    w = WORKLOADS["stream"]
    dev = torch.device("cuda")
    s0 = make_state(w, device=dev)
    calls = [make_inputs(w, call=c, device=dev) for c in range(2)]
    outs_a = [torch.empty_like(c[0]) for c in calls]
    outs_b = [torch.empty_like(c[0]) for c in calls]
    # reference: gla_forward, state carried from call 0 into call 1
    state_a = s0.clone()
    for (q, k, v, g), out in zip(calls, outs_a):
        gla.gla_forward(q, k, v, g, state_a, state_a, out, w.B, w.H, 1, w.tokens_per_frame,
                        w.d, w.eps)
    state_b = s0.clone()
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for (q, k, v, g), out in zip(calls, outs_b):
        gla.gla_forward_noalloc(q, k, v, g, state_b, state_b, out, w.B, w.H, 1,
                                w.tokens_per_frame, w.d, w.eps)
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    for call in range(2):
        _close(outs_b[call], outs_a[call], "call %d out" % call)
    _close(state_b, state_a, "state after two calls")
    assert free1 >= free0, "gla_forward_noalloc took device memory (%d -> %d)" % (free0, free1)
    assert gla.gla_device_fault() == 0


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
