"""Parity of gla_forward_rope (through the C ABI) with the fp64 RoPE oracle.

Tolerance as the plain layer: max|gpu - oracle| <= 1e-2 max|oracle| and
rel-L2 <= 5e-3, on out and state_out.  Small shapes for every head dim (the
three feature blocks in several splits, grids narrower and wider than a
tile, frame offsets, random initial state, ragged tails) are compared in
full; the 720p-5s layer (46 x 80 latent grid) runs at full size and is
compared on sampled (batch, head) slices.
"""

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, make_inputs, make_state

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
    err = np.abs(gpu - ref)
    scale = np.abs(ref).max()
    l2 = np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-300)
    assert err.max() <= TOL_MAX * scale, "%s: max err %.3e > %.1e * %.3e" % (what, err.max(),
                                                                            TOL_MAX, scale)
    assert l2 <= TOL_L2, "%s: rel L2 %.3e > %.1e" % (what, l2, TOL_L2)


def case(B, H, F, T, d, state, seed, k_scaled=False):
    w = WORKLOADS["tiny"].with_(B=B, H=H, frames=F, tokens_per_frame=T, d=d, k_scaled=k_scaled,
                                random_state_in=state)
    q, k, v, g = make_inputs(w, seed=seed)
    s = make_state(w, seed=seed)
    if s is not None:
        s[..., d] = s[..., d].abs() + 1.0
    return q, k, v, g, s


def run_gpu(q, k, v, g, s, rope):
    dev = torch.device("cuda")
    qd, kd, vd, gd = (x.to(dev) for x in (q, k, v, g))
    sd = None if s is None else s.to(dev)
    out, so = gla().forward_rope(qd, kd, vd, gd, rope, state_in=sd, eps=EPS)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), so.cpu().numpy()


SMALL = [
    # B, H, F, T, d, state, dims, grid_w, frame_offset, theta
    (1, 2, 3, 200, 128, True, (32, 48, 48), 20, 0, 10000.0),
    (2, 3, 2, 300, 128, False, (32, 48, 48), 80, 5, 10000.0),
    (1, 2, 4, 37, 64, True, (16, 24, 24), 7, 2, 100.0),
    (1, 4, 2, 129, 32, False, (8, 8, 16), 16, 0, 50.0),
    (1, 1, 5, 64, 128, True, (128, 0, 0), 8, 3, 10000.0),
    (2, 2, 2, 256, 128, False, (0, 64, 64), 3, 0, 1000.0),
    (1, 149, 1, 150, 64, True, (16, 24, 24), 10, 1, 10000.0),   # more units than CTAs
]


@pytest.mark.parametrize("B,H,F,T,d,state,dims,grid_w,offset,theta", SMALL)
def test_small_shapes_full_compare(B, H, F, T, d, state, dims, grid_w, offset, theta):
    q, k, v, g, s = case(B, H, F, T, d, state, seed=7000 + B * 100 + H * 10 + F + T + d)
    rope = gla().rope_config(grid_w, dims, offset, theta)
    out, so = run_gpu(q, k, v, g, s, rope)
    ref, sref = oracle.gla_rope_forward(q, k, v, g, F, grid_w, offset, dims, theta, s, EPS)
    assert_close(out, ref, "out")
    assert_close(so, sref, "state_out")


def test_zero_angles_match_plain_layer():
    """One frame at offset 0 with only a temporal block: every angle is zero."""
    q, k, v, g, s = case(1, 3, 1, 300, 128, True, 31)
    out, so = run_gpu(q, k, v, g, s, gla().rope_config(80, (128, 0, 0), 0))
    ref, sref = oracle.gla_forward(q, k, v, g, 1, s, EPS)
    assert_close(out, ref, "out")
    assert_close(so, sref, "state_out")


def test_streamed_calls_with_offsets():
    q, k, v, g, s = case(1, 2, 4, 160, 128, True, 41)
    dims, gw = (32, 48, 48), 40
    full, s_full = run_gpu(q, k, v, g, s, gla().rope_config(gw, dims, 0))
    n = 2 * 160
    o1, s1 = run_gpu(q[:, :n], k[:, :n], v[:, :n], g[:, :2], s, gla().rope_config(gw, dims, 0))
    o2, s2 = run_gpu(q[:, n:], k[:, n:], v[:, n:], g[:, 2:], torch.from_numpy(s1),
                     gla().rope_config(gw, dims, 2))
    assert_close(np.concatenate([o1, o2], axis=1), full, "out")
    assert_close(s2, s_full, "state_out")


def test_full_size_720p_5s_sampled_heads():
    w = WORKLOADS["720p-5s"]
    dev = torch.device("cuda")
    q, k, v, g = make_inputs(w, device=dev)
    rope = gla().rope_config(80, (32, 48, 48), 0, 10000.0)
    out, so = gla().forward_rope(q, k, v, g, rope, eps=w.eps)
    torch.cuda.synchronize()
    for b, h in [(0, 0), (1, 17)]:
        sl = lambda x: x[b, :, h].float().cpu().numpy()  # noqa: E731
        ref, sref = oracle.gla_rope_head(sl(q), sl(k), sl(v), g[b, :, h].cpu().numpy(),
                                         w.tokens_per_frame, 80, 0, (32, 48, 48), 10000.0, None,
                                         w.eps)
        assert_close(sl(out), ref, "out[b=%d,h=%d]" % (b, h))
        assert_close(so[b, h].cpu().numpy(), sref, "state_out[b=%d,h=%d]" % (b, h))
