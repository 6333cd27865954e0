"""Parity of gla_forward_gdn (through the C ABI) with the fp64 delta-rule oracle.

Tolerance as the plain layer (max|err| <= 1e-2 max|oracle|, rel-L2 <= 5e-3)
on out and state_out.  Keys are drawn with the 1/sqrt(d T) scale the SANA-WM
pages give for the delta rule (the recurrence contracts); small shapes for
every head dim cover ragged tails, units split over several increment CTAs
(their Gram partials summed by the scan), more units than CTAs, random
initial state, tokenless frames; the 720p-5s shape runs at full size and is
compared on sampled (batch, head) slices.
"""

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, gdn_workload, make_beta, make_inputs, make_state

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


def assert_close(gpu, ref, what=""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, what
    assert np.all(np.isfinite(gpu)), what + ": non-finite values"
    if ref.size == 0:
        return
    err = np.abs(gpu - ref)
    scale = np.abs(ref).max()
    l2 = np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-300)
    assert err.max() <= TOL_MAX * scale, "%s: max err %.3e > %.1e * %.3e" % (what, err.max(),
                                                                            TOL_MAX, scale)
    assert l2 <= TOL_L2, "%s: rel L2 %.3e > %.1e" % (what, l2, TOL_L2)


def case(B, H, F, T, d, state, seed):
    w = gdn_workload(WORKLOADS["tiny"].with_(B=B, H=H, frames=F, tokens_per_frame=T, d=d,
                                             g_mu=2.0, g_sigma=1.0, random_state_in=state))
    q, k, v, g = make_inputs(w, seed=seed)
    bl = make_beta(w, seed=seed)
    s = make_state(w, seed=seed)
    if s is not None:
        s[..., d] = s[..., d].abs() + 1.0
    return q, k, v, g, bl, s


def run_gpu(q, k, v, g, bl, s):
    dev = torch.device("cuda")
    qd, kd, vd, gd, bd = (x.to(dev) for x in (q, k, v, g, bl))
    sd = None if s is None else s.to(dev)
    out, so = gla().forward_gdn(qd, kd, vd, gd, bd, state_in=sd, eps=EPS)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), so.cpu().numpy()


SMALL = [
    # B, H, F, T, d, random state
    (1, 2, 4, 16, 32, False),
    (2, 3, 3, 37, 64, True),
    (1, 2, 3, 200, 128, True),
    (2, 2, 5, 128, 128, False),
    (1, 1, 1, 1, 128, True),
    (1, 4, 6, 129, 32, True),
    (1, 37, 2, 400, 128, True),     # units split over two CTAs
    (2, 40, 3, 64, 128, False),     # more units than CTAs
    (1, 1, 2, 5120, 128, True),     # each unit split over 40 CTAs (40 partials summed)
    (1, 3, 7, 255, 64, True),
]


@pytest.mark.parametrize("B,H,F,T,d,state", SMALL)
def test_small_shapes_full_compare(B, H, F, T, d, state):
    q, k, v, g, bl, s = case(B, H, F, T, d, state, seed=9000 + B * 100 + H * 10 + F + T + d)
    out, so = run_gpu(q, k, v, g, bl, s)
    ref, sref = oracle.gla_gdn_forward(q, k, v, g, bl, F, s, EPS)
    assert_close(out, ref, "out")
    assert_close(so, sref, "state_out")


def test_beta_zero_only_decays():
    q, k, v, g, bl, s = case(1, 2, 3, 100, 128, True, 21)
    out, so = run_gpu(q, k, v, g, torch.full_like(bl, -float("inf")), s)
    a = torch.sigmoid(g.double())
    want = s.double() * torch.prod(a, dim=1)[:, :, None, None]
    assert_close(so, want.numpy(), "state_out")


def test_no_tokens_and_no_frames():
    q, k, v, g, bl, s = case(1, 2, 3, 0, 128, True, 23)
    out, so = run_gpu(q, k, v, g, bl, s)
    a = torch.sigmoid(g.double())
    assert_close(so, (s.double() * torch.prod(a, dim=1)[:, :, None, None]).numpy(), "state_out")
    q0 = torch.empty(1, 0, 2, 128, dtype=torch.bfloat16)
    g0 = torch.empty(1, 0, 2)
    out, so = run_gpu(q0, q0, q0, g0, g0, s)
    np.testing.assert_array_equal(so, s.numpy())


def test_full_size_720p_5s_sampled_heads():
    w = gdn_workload(WORKLOADS["720p-5s"])
    dev = torch.device("cuda")
    q, k, v, g = make_inputs(w, device=dev)
    bl = make_beta(w, device=dev)
    out, so = gla().forward_gdn(q, k, v, g, bl, eps=w.eps)
    torch.cuda.synchronize()
    for b, h in [(0, 0), (1, 17)]:
        sl = lambda x: x[b, :, h].float().cpu().numpy()  # noqa: E731
        ref, sref = oracle.gla_gdn_head(sl(q), sl(k), sl(v), g[b, :, h].cpu().numpy(),
                                        bl[b, :, h].cpu().numpy(), w.tokens_per_frame, None, w.eps)
        assert_close(sl(out), ref, "out[b=%d,h=%d]" % (b, h))
        assert_close(so[b, h].cpu().numpy(), sref, "state_out[b=%d,h=%d]" % (b, h))


def test_streamed_calls_match_one_call():
    """Chunking through state_out -> state_in equals one call (the delta rule
    depends on the carried state through M_f S_{f-1})."""
    q, k, v, g, bl, s = case(1, 3, 5, 150, 128, True, 31)
    full, s_full = run_gpu(q, k, v, g, bl, s)
    n = 2 * 150
    o1, s1 = run_gpu(q[:, :n], k[:, :n], v[:, :n], g[:, :2], bl[:, :2], s)
    o2, s2 = run_gpu(q[:, n:], k[:, n:], v[:, n:], g[:, 2:], bl[:, 2:], torch.from_numpy(s1))
    assert_close(np.concatenate([o1, o2], axis=1), full, "out")
    assert_close(s2, s_full, "state_out")
