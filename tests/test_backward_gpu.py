"""Parity of gla_backward (through the C ABI) with the fp64 gradient oracle.

Same tolerance as the forward, applied to every gradient:
    max|gpu - oracle| <= 1e-2 * max|oracle|  and  ||gpu - oracle||_2 <= 5e-3 * ||oracle||_2
to dq, dk, dv (bf16), dgate_logits and dstate_in (fp32).  Small d = 128 shapes
(ragged tails, several tiles per frame, units split over CTAs, more units than
CTAs, random initial state and state gradient) are compared in full; the
720p-5s layer runs at full size and is compared on sampled (batch, head)
slices, which the oracle computes one by one.
"""

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, make_grads, make_inputs, make_state

pytestmark = pytest.mark.gpu

TOL_MAX = 1e-2
TOL_L2 = 5e-3
EPS = 1e-6


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


def gla():
    import gated_linear_attention_frame_b200 as g

    return g


def assert_close(gpu, ref, what="", atol=0.0, widen=1.0):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, what
    assert np.all(np.isfinite(gpu)), what + ": non-finite values"
    err = np.abs(gpu - ref)
    scale = np.abs(ref).max() if ref.size else 0.0
    if err.size == 0:
        return
    l2 = np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-300)
    assert err.max() <= widen * TOL_MAX * scale + atol, "%s: max err %.3e > %.1e * %.3e" % (
        what, err.max(), widen * TOL_MAX, scale)
    if atol == 0.0:
        assert l2 <= widen * TOL_L2, "%s: rel L2 %.3e > %.1e" % (what, l2, widen * TOL_L2)


def case(B, H, F, T, state, dstate, seed, g_mu=2.0, g_sigma=1.0, k_scaled=False):
    w = WORKLOADS["tiny"].with_(B=B, H=H, frames=F, tokens_per_frame=T, d=128, g_mu=g_mu,
                                g_sigma=g_sigma, k_scaled=k_scaled, random_state_in=state)
    q, k, v, g = make_inputs(w, seed=seed)
    s = make_state(w, seed=seed)
    if s is not None:
        s[..., 128] = s[..., 128].abs() + 1.0  # a positive normaliser column
    dout, ds = make_grads(w, seed=seed, dstate_out=dstate)
    return w, q, k, v, g, s, dout, ds


def run_gpu(q, k, v, g, s, dout, ds, frames, want_ds_in=True):
    dev = torch.device("cuda")
    args = [None if x is None else x.to(dev) for x in (q, k, v, g, dout, s, ds)]
    qd, kd, vd, gd, dod, sd, dsd = args
    r = gla().backward(qd, kd, vd, gd, dod, state_in=sd, dstate_out=dsd, eps=EPS,
                       want_dstate_in=want_ds_in)
    torch.cuda.synchronize()
    return [None if x is None else x.float().cpu().numpy() for x in r]


def reference(q, k, v, g, s, dout, ds, frames, want_ds_in=True):
    s_ref = s
    if s is None and want_ds_in:
        s_ref = torch.zeros(q.shape[0], q.shape[2], 128, 129)
    return oracle.gla_backward(q, k, v, g, frames, dout, s_ref, ds, EPS)


def compare_all(got, ref, label=""):
    """Every gradient to the spec's tolerance, with no widening."""
    names = ("dq", "dk", "dv", "dgate", "dstate_in")
    for n, a, b in zip(names, got, ref):
        if b is None:
            assert a is None, n
            continue
        assert_close(a, b, label + n)


SMALL = [
    # B, H, F, T, random state_in, dstate_out
    (1, 2, 3, 200, True, True),
    (2, 3, 2, 128, False, False),
    (1, 1, 1, 1, True, True),
    # frames of one to three tokens: dk_t = 1[k_t > 0] ([v_t | 1] G_f^T) cancels
    # most there (out_t stays near v_t), the case that needs G_f in hi/lo parts
    (1, 1, 3, 1, True, True),
    (1, 2, 6, 3, True, False),
    # from a zero state dq cancels exactly in the first frame of one-token
    # frames (out = v there, whatever q): the case that needs dq from dout
    # against S_f in hi/lo parts
    (1, 2, 3, 1, False, True),
    (1, 1, 5, 1, False, False),
    (1, 3, 3, 2, False, True),
    (1, 4, 2, 2, False, False),
    (1, 2, 5, 300, False, True),
    (1, 1, 2, 700, True, False),
    (1, 3, 4, 64, True, True),
    # a unit's tiles split over two CTAs (2 tiles per CTA on 148 SMs)
    (1, 37, 2, 400, True, True),
    # more units than CTAs, and a tail of one unit
    (2, 40, 3, 64, False, True),
    (1, 149, 1, 200, True, False),
]


@pytest.mark.parametrize("B,H,F,T,state,dstate", SMALL)
def test_small_shapes_full_compare(B, H, F, T, state, dstate):
    seed = 5000 + B * 100 + H * 10 + F + T
    w, q, k, v, g, s, dout, ds = case(B, H, F, T, state, dstate, seed)
    got = run_gpu(q, k, v, g, s, dout, ds, F)
    ref = reference(q, k, v, g, s, dout, ds, F)
    compare_all(got, ref)


def test_scaled_keys_slow_decay():
    w, q, k, v, g, s, dout, ds = case(1, 2, 6, 500, False, False, 77, g_mu=4.0, g_sigma=0.5,
                                      k_scaled=True)
    compare_all(run_gpu(q, k, v, g, s, dout, ds, 6), reference(q, k, v, g, s, dout, ds, 6))


@pytest.mark.parametrize("glogit", [30.0, -30.0])
def test_gate_extremes(glogit):
    """a = 1 (no decay) and a = 0 (frame-local) across the whole sequence."""
    w, q, k, v, g, s, dout, ds = case(1, 2, 3, 150, True, True, 91)
    g = torch.full_like(g, glogit)
    got = run_gpu(q, k, v, g, s, dout, ds, 3)
    ref = reference(q, k, v, g, s, dout, ds, 3)
    compare_all(got[:3] + [None] + got[4:], ref[:3] + (None,) + ref[4:])
    # a (1 - a) is ~1e-13 in fp64 and exactly 0 in fp32 at a = 1: absolute bound
    scale = max(np.abs(ref[3]).max(), 1e-30)
    assert np.abs(got[3] - ref[3]).max() <= TOL_MAX * scale + 1e-9


def test_no_tokens_only_decays():
    """tokens_per_frame = 0: dq/dk/dv are empty, dgate and dstate_in remain."""
    w, q, k, v, g, s, dout, ds = case(1, 2, 4, 0, True, True, 13)
    got = run_gpu(q, k, v, g, s, dout, ds, 4)
    ref = reference(q, k, v, g, s, dout, ds, 4)
    assert got[0].size == 0
    assert_close(got[3], ref[3], "dgate")
    assert_close(got[4], ref[4], "dstate_in")


def test_no_frames_passes_state_gradient():
    dev = torch.device("cuda")
    q = torch.empty(1, 0, 2, 128, dtype=torch.bfloat16, device=dev)
    g = torch.empty(1, 0, 2, device=dev)
    ds = torch.randn(1, 2, 128, 129, device=dev, generator=torch.Generator(dev).manual_seed(3))
    r = gla().backward(q, q, q, g, q, state_in=None, dstate_out=ds, eps=EPS)
    torch.cuda.synchronize()
    assert torch.equal(r[4], ds)
    r = gla().backward(q, q, q, g, q, state_in=None, dstate_out=None, eps=EPS)
    torch.cuda.synchronize()
    assert torch.count_nonzero(r[4]) == 0


def test_deterministic():
    w, q, k, v, g, s, dout, ds = case(1, 37, 2, 400, True, True, 4242)
    a = run_gpu(q, k, v, g, s, dout, ds, 2)
    b = run_gpu(q, k, v, g, s, dout, ds, 2)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_dstate_in_not_requested():
    w, q, k, v, g, s, dout, ds = case(1, 2, 3, 100, True, True, 8)
    got = run_gpu(q, k, v, g, s, dout, ds, 3, want_ds_in=False)
    ref = reference(q, k, v, g, s, dout, ds, 3)
    assert got[4] is None
    compare_all(got[:4], ref[:4])


def test_matches_streamed_calls():
    """Two calls chained through the state: the gradient of the pair equals the
    second call's backward fed into the first's dstate_out."""
    w, q, k, v, g, s, dout, ds = case(1, 2, 4, 160, True, True, 99)
    dev = torch.device("cuda")
    qd, kd, vd, gd, dod, sd, dsd = (x.to(dev) for x in (q, k, v, g, dout, s, ds))
    full = gla().backward(qd, kd, vd, gd, dod, state_in=sd, dstate_out=dsd, eps=EPS)
    n = 2 * 160
    _, s_mid = gla().forward(qd[:, :n].contiguous(), kd[:, :n].contiguous(),
                             vd[:, :n].contiguous(), gd[:, :2].contiguous(), state_in=sd, eps=EPS)
    second = gla().backward(qd[:, n:].contiguous(), kd[:, n:].contiguous(), vd[:, n:].contiguous(),
                            gd[:, 2:].contiguous(), dod[:, n:].contiguous(), state_in=s_mid,
                            dstate_out=dsd, eps=EPS)
    first = gla().backward(qd[:, :n].contiguous(), kd[:, :n].contiguous(), vd[:, :n].contiguous(),
                           gd[:, :2].contiguous(), dod[:, :n].contiguous(), state_in=sd,
                           dstate_out=second[4], eps=EPS)
    torch.cuda.synchronize()
    for i, name in enumerate(("dq", "dk", "dv")):
        cat = torch.cat([first[i], second[i]], dim=1)
        assert_close(cat.float().cpu().numpy(), full[i].float().cpu().numpy(), name)
    assert_close(torch.cat([first[3], second[3]], dim=1).cpu().numpy(), full[3].cpu().numpy(),
                 "dgate")
    assert_close(first[4].cpu().numpy(), full[4].cpu().numpy(), "dstate_in")


@pytest.mark.parametrize("heads", [[(0, 0), (1, 23)]])
def test_full_size_720p_5s_sampled_heads(heads):
    w = WORKLOADS["720p-5s"]
    dev = torch.device("cuda")
    q, k, v, g = make_inputs(w, device=dev)
    dout, _ = make_grads(w, device=dev)
    dq, dk, dv, dg, _ = gla().backward(q, k, v, g, dout, eps=w.eps, want_dstate_in=False)
    torch.cuda.synchronize()
    T = w.tokens_per_frame
    for b, h in heads:
        sl = lambda x: x[b, :, h].float().cpu().numpy()  # noqa: E731
        ref = oracle.gla_backward_head_manual(sl(q), sl(k), sl(v), g[b, :, h].cpu().numpy(), T,
                                              sl(dout), None, None, w.eps)
        for name, got, r in zip(("dq", "dk", "dv", "dgate"),
                                (sl(dq), sl(dk), sl(dv), dg[b, :, h].cpu().numpy()), ref[:4]):
            assert_close(got, r, "%s[b=%d,h=%d]" % (name, b, h))
