"""Failure paths of the library on the GPU, made without a GPU fault.

  * Workspace allocation failure: a host-side hook (gla_inject_alloc_failure)
    makes the next allocation fail; the call returns GLA_ERR_ALLOC and
    enqueues nothing (out and state_out keep their sentinel), and the next
    call is parity-green.
  * A bounded device wait that runs out: the wait limit is lowered to a few
    milliseconds (gla_set_wait_limit_ns) and the state-increment kernel's
    first CTA withholds the loads of one tile (gla_inject_stall), so nothing
    ever arrives on that tile's barrier.  The kernel must give up, report bit
    0 through gla_device_fault, let its copies land, free its tensor memory
    and return; the call's later kernels then finish on their own; the next
    normal call (whose kernels allocate tensor memory on the same SMs again)
    must be parity-green with no fault.
  * Workspace retention: after gla_trim_workspace the memory the pool kept
    returns to the device; with a retention of 0 it returns at the caller's
    synchronisation.
"""

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

TOL_MAX = 1e-2
TOL_L2 = 5e-3
SENTINEL = 12345.0


@pytest.fixture(scope="module")
def gla():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gated_linear_attention_frame_b200.build import build

    build()
    import gated_linear_attention_frame_b200 as g

    g.load_library()
    g.gla_device_fault()  # start from a clear fault word
    yield g
    g.gla_set_wait_limit_ns(0)
    g.gla_inject_stall(-1)
    g.gla_inject_alloc_failure(0)


def _case(B=1, H=2, F=3, T=300, d=128):
    w = WORKLOADS["tiny"].with_(B=B, H=H, d=d, frames=F, tokens_per_frame=T)
    q, k, v, g = make_inputs(w)
    dev = torch.device("cuda")
    return w, (q, k, v, g), tuple(x.to(dev) for x in (q, k, v, g))


def _call(gla, w, dev_in):
    q, k, v, g = dev_in
    out = torch.full_like(q, SENTINEL)
    state = torch.full((w.B, w.H, w.d, w.d + 1), SENTINEL, device=q.device)
    gla.gla_forward(q, k, v, g, None, state, out, w.B, w.H, w.frames, w.tokens_per_frame, w.d,
                    w.eps)
    return out, state


def _parity(w, host_in, out, state):
    q, k, v, g = host_in
    ref, sref = oracle.gla_forward(q, k, v, g, w.frames, None, w.eps)
    for name, got, r in (("out", out, ref), ("state", state, sref)):
        got = got.double().cpu().numpy()
        assert np.all(np.isfinite(got)), name
        err = np.abs(got - r).max()
        assert err <= TOL_MAX * np.abs(r).max(), "%s: max err %.3e" % (name, err)
        l2 = np.linalg.norm(got - r) / np.linalg.norm(r)
        assert l2 <= TOL_L2, "%s: rel L2 %.3e" % (name, l2)


def test_alloc_failure_returns_status_and_enqueues_nothing(gla):
    w, host_in, dev_in = _case()
    gla.gla_inject_alloc_failure(1)
    q, k, v, g = dev_in
    out = torch.full_like(q, SENTINEL)
    state = torch.full((w.B, w.H, w.d, w.d + 1), SENTINEL, device=q.device)
    with pytest.raises(gla.GLAError) as ei:
        gla.gla_forward(q, k, v, g, None, state, out, w.B, w.H, w.frames, w.tokens_per_frame,
                        w.d, w.eps)
    assert ei.value.status == gla.GLA_ERR_ALLOC
    torch.cuda.synchronize()
    assert bool((out == SENTINEL).all()) and bool((state == SENTINEL).all()), \
        "a call that failed its allocation wrote its outputs"
    # the backward pass takes its workspace the same way
    gla.gla_inject_alloc_failure(1)
    with pytest.raises(gla.GLAError) as ei:
        gla.backward(q, k, v, g, q, eps=w.eps)
    assert ei.value.status == gla.GLA_ERR_ALLOC
    # the hook is spent: the next call runs
    out, state = _call(gla, w, dev_in)
    torch.cuda.synchronize()
    assert gla.gla_device_fault() == 0
    _parity(w, host_in, out, state)


@pytest.mark.parametrize("tile", [0, 1])
def test_wait_that_runs_out_is_reported_and_recovered(gla, tile):
    # 2 heads x 3 frames x 300 tokens: 18 tiles on 18 CTAs, one each; 24 heads
    # x 3 frames x 700 tokens: 432 tiles on (at most) 148 CTAs, so CTA 0 holds
    # two or more and tile 1 is a later one of its sequence
    w, host_in, dev_in = _case(H=2 if tile == 0 else 24, T=300 if tile == 0 else 700)
    try:
        gla.gla_set_wait_limit_ns(5_000_000)  # 5 ms
        gla.gla_inject_stall(tile)
        out, state = _call(gla, w, dev_in)
        torch.cuda.synchronize()  # the call's kernels returned
        fault = gla.gla_device_fault()
    finally:
        gla.gla_set_wait_limit_ns(0)
        gla.gla_inject_stall(-1)
    assert fault & 1, "the increment kernel did not report its wait (fault word %#x)" % fault
    # a normal call afterwards: tensor memory free again, results correct
    out, state = _call(gla, w, dev_in)
    torch.cuda.synchronize()
    assert gla.gla_device_fault() == 0
    _parity(w, host_in, out, state)


def test_workspace_pool_returns_memory(gla):
    # half of the 720p-5s layer: about 55 MB of workspace
    w, _, dev_in = _case(B=1, H=24, F=21, T=3680)
    out = torch.empty_like(dev_in[0])
    state = torch.empty(w.B, w.H, w.d, w.d + 1, device=out.device)
    ws_bytes = (w.B * w.H * w.frames * 6 + 148 * 4) * (w.d + 1) * w.d
    q, k, v, g = dev_in

    def call():
        gla.gla_forward(q, k, v, g, None, state, out, w.B, w.H, w.frames, w.tokens_per_frame,
                        w.d, w.eps)
        torch.cuda.synchronize()

    try:
        gla.gla_set_workspace_retention(2 ** 64 - 1)  # the default: keep everything
        gla.gla_trim_workspace()
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        call()
        free1 = torch.cuda.mem_get_info()[0]
        assert free0 - free1 >= ws_bytes // 2, "the pool kept nothing (%d -> %d)" % (free0, free1)
        gla.gla_trim_workspace()
        torch.cuda.synchronize()
        free2 = torch.cuda.mem_get_info()[0]
        assert free2 >= free0 - (4 << 20), "trim left %d bytes mapped" % (free0 - free2)
        # retention 0: the workspace goes back at the synchronisation itself
        gla.gla_set_workspace_retention(0)
        call()
        free3 = torch.cuda.mem_get_info()[0]
        assert free3 >= free0 - (4 << 20), "retention 0 kept %d bytes" % (free0 - free3)
    finally:
        gla.gla_set_workspace_retention(2 ** 64 - 1)
    assert gla.gla_device_fault() == 0
