"""The training pair gla_forward_train / gla_backward_saved through the C ABI.

The training forward writes the per-frame states it computes into a
caller-owned context; the backward from that context skips the recompute of
the states.  Both run the same kernels on the same values as gla_forward and
gla_backward, so they are checked against them bit for bit:
  * out and state_out of gla_forward_train equal gla_forward's (single-frame
    calls included, where gla_forward folds the scan step into the increment
    kernel and the training forward runs the scan);
  * every gradient of gla_backward_saved equals gla_backward's;
  * the context is only read by the backward;
and one case against the fp64 gradient oracle at the parity tolerance.
"""

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, make_grads, make_inputs, make_state

pytestmark = pytest.mark.gpu

EPS = 1e-6
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


def _case(B, H, F, T, state, dstate, seed):
    w = WORKLOADS["tiny"].with_(B=B, H=H, frames=F, tokens_per_frame=T, d=128,
                                random_state_in=state)
    q, k, v, g = make_inputs(w, seed=seed)
    s = make_state(w, seed=seed)
    if s is not None:
        s[..., 128] = s[..., 128].abs() + 1.0  # a positive normaliser column
    dout, ds = make_grads(w, seed=seed, dstate_out=dstate)
    return w, q, k, v, g, s, dout, ds


SHAPES = [
    # B, H, frames, T, random state_in, dstate_out
    (1, 2, 3, 200, True, True),     # ragged tiles, several frames
    (2, 3, 2, 128, False, False),
    (1, 1, 1, 300, True, False),    # one frame: the forward's fold path vs the scan
    (8, 24, 1, 260, True, True),    # one frame, units split over CTAs
    (1, 2, 5, 3, False, True),      # frames of a few tokens
    (2, 24, 7, 700, True, True),    # more units than CTAs
]


@pytest.mark.parametrize("B,H,F,T,state,dstate", SHAPES)
def test_training_pair_equals_forward_and_backward(gla, B, H, F, T, state, dstate):
    w, q, k, v, g, s, dout, ds = _case(B, H, F, T, state, dstate, seed=7000 + B + H + F + T)
    dev = torch.device("cuda")
    q, k, v, g, dout = (x.to(dev) for x in (q, k, v, g, dout))
    s = None if s is None else s.to(dev)
    ds = None if ds is None else ds.to(dev)
    out_a, st_a = gla.forward(q, k, v, g, state_in=s, eps=EPS)
    out_b, st_b, saved = gla.forward_train(q, k, v, g, state_in=s, eps=EPS)
    torch.cuda.synchronize()
    assert saved.numel() == gla.gla_saved_bytes(B, H, F, T, 128)
    assert torch.equal(out_b, out_a), "training forward: out differs"
    assert torch.equal(st_b, st_a), "training forward: state_out differs"
    before = saved.clone()
    ra = gla.backward(q, k, v, g, dout, state_in=s, dstate_out=ds, eps=EPS)
    rb = gla.backward(q, k, v, g, dout, state_in=s, dstate_out=ds, eps=EPS, saved=saved)
    torch.cuda.synchronize()
    for name, a, b in zip(("dq", "dk", "dv", "dgate", "dstate_in"), ra, rb):
        assert torch.equal(b, a), "saved backward: %s differs" % name
    assert torch.equal(saved, before), "the backward wrote into the saved context"
    assert gla.gla_device_fault() == 0


def test_training_pair_against_oracle(gla):
    B, H, F, T = 1, 2, 3, 200
    w, q, k, v, g, s, dout, ds = _case(B, H, F, T, True, True, seed=7100)
    dev = torch.device("cuda")
    qd, kd, vd, gd, dod, sd, dsd = (x.to(dev) for x in (q, k, v, g, dout, s, ds))
    _, _, saved = gla.forward_train(qd, kd, vd, gd, state_in=sd, eps=EPS)
    got = gla.backward(qd, kd, vd, gd, dod, state_in=sd, dstate_out=dsd, eps=EPS, saved=saved)
    torch.cuda.synchronize()
    ref = oracle.gla_backward(q, k, v, g, F, dout, s, ds, EPS)
    for name, x, r in zip(("dq", "dk", "dv", "dgate", "dstate_in"), got, ref):
        x = x.double().cpu().numpy()
        r = np.asarray(r, dtype=np.float64)
        assert x.shape == r.shape, name
        err = np.abs(x - r).max()
        assert err <= TOL_MAX * np.abs(r).max(), "%s: max err %.3e" % (name, err)
        l2 = np.linalg.norm(x - r) / np.linalg.norm(r)
        assert l2 <= TOL_L2, "%s: rel L2 %.3e" % (name, l2)
