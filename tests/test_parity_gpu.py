"""Parity of the CUDA library (through its C ABI) with the fp64 CPU oracle.

Tolerance (bf16 inputs, bf16 output, fp32 state):
    max|gpu - oracle| <= 1e-2 * max|oracle|   and   ||gpu - oracle||_2 <= 5e-3 * ||oracle||_2
applied to `out` and to `state_out`.

Small shapes (ragged tails, several tiles per frame, every head dim, gate
extremes, random initial state) are compared element by element in full.  The
full-size layer workloads run exactly as the benchmark launches them and are
compared on sampled (batch, head) slices, which the oracle computes one by one
(heads are independent).  The streaming workload carries the state through 64
consecutive calls on both sides.
"""

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, make_inputs, make_state

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
    # no kernel of the whole module may have given up a bounded wait
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
    return err.max() / max(scale, 1e-300), l2


def run_gpu(q, k, v, g, s_in, frames, eps=1e-6, state_out=True):
    B, N, H, d = q.shape
    T = N // frames if frames else 0
    dev = torch.device("cuda")
    qd, kd, vd, gd = (x.to(dev) for x in (q, k, v, g))
    sd = None if s_in is None else s_in.to(dev)
    out = torch.empty_like(qd)
    so = torch.empty(B, H, d, d + 1, device=dev, dtype=torch.float32) if state_out else None
    gla().gla_forward(qd, kd, vd, gd, sd, so, out, B, H, frames, T, d, eps)
    torch.cuda.synchronize()
    return out, so


def small_case(B, H, F, T, d, state, seed, g_mu=2.0, g_sigma=1.0, k_scaled=False):
    w = WORKLOADS["tiny"].with_(B=B, H=H, frames=F, tokens_per_frame=T, d=d, g_mu=g_mu,
                                g_sigma=g_sigma, k_scaled=k_scaled, random_state_in=state)
    q, k, v, g = make_inputs(w, seed=seed)
    s = make_state(w, seed=seed)
    if s is not None:
        s[..., d] = s[..., d].abs() + 1.0  # a positive normaliser column
    return w, q, k, v, g, s


SMALL = [
    # B, H, F, T, d, random state
    (1, 2, 4, 16, 32, False),
    (2, 3, 3, 37, 64, True),
    (1, 2, 2, 200, 128, True),
    (2, 2, 5, 128, 128, False),
    (1, 1, 1, 1, 128, False),
    (1, 4, 6, 129, 32, True),
    (3, 5, 2, 300, 64, False),
    (1, 3, 7, 255, 128, True),
    (2, 1, 3, 1000, 128, False),
    (1, 2, 9, 77, 64, True),
    # schedule edges on 148 SMs: a tail of one unit, an exact multiple of the
    # CTA count, a tail with fewer tiles than CTAs
    (1, 149, 1, 200, 64, True),
    (2, 37, 4, 130, 32, False),
    (1, 150, 1, 1, 32, False),
]


@pytest.mark.parametrize("B,H,F,T,d,state", SMALL)
def test_small_shapes_full_compare(B, H, F, T, d, state):
    w, q, k, v, g, s = small_case(B, H, F, T, d, state, seed=1000 + B * 100 + H * 10 + F + T + d)
    out, so = run_gpu(q, k, v, g, s, F)
    ref, sref = oracle.gla_forward(q, k, v, g, F, s, 1e-6)
    assert_close(out.float().cpu().numpy(), ref, "out")
    assert_close(so.cpu().numpy(), sref, "state_out")


def test_tiny_workload():
    w = WORKLOADS["tiny"]
    q, k, v, g = make_inputs(w)
    out, so = run_gpu(q, k, v, g, None, w.frames, w.eps)
    ref, sref = oracle.gla_forward(q, k, v, g, w.frames, None, w.eps)
    assert_close(out.float().cpu().numpy(), ref, "out")
    assert_close(so.cpu().numpy(), sref, "state_out")


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("gate", ["a=1", "a=0", "mixed"])
def test_gate_extremes(d, gate):
    F, T = 4, 70
    w, q, k, v, g, s = small_case(2, 2, F, T, d, True, seed=77 + d)
    if gate == "a=1":
        g = torch.full_like(g, float("inf"))
    elif gate == "a=0":
        g = torch.full_like(g, float("-inf"))
    else:
        g[:, 0] = float("inf")
        g[:, 1] = float("-inf")
    out, so = run_gpu(q, k, v, g, s, F)
    ref, sref = oracle.gla_forward(q, k, v, g, F, s, 1e-6)
    assert_close(out.float().cpu().numpy(), ref, "out")
    assert_close(so.cpu().numpy(), sref, "state_out")


def test_chunking_invariance_gpu():
    """One call over all frames == frame-by-frame calls threaded through
    state_in/state_out == an uneven split (block KV cache reuse)."""
    F, T, d = 6, 300, 128
    w, q, k, v, g, s = small_case(2, 3, F, T, d, True, seed=5)
    out_all, s_all = run_gpu(q, k, v, g, s, F)
    for splits in ([1] * F, [2, 4], [5, 1]):
        state = s
        outs = []
        f0 = 0
        for n in splits:
            rows = slice(f0 * T, (f0 + n) * T)
            o, state = run_gpu(q[:, rows].contiguous(), k[:, rows].contiguous(),
                               v[:, rows].contiguous(), g[:, f0:f0 + n].contiguous(),
                               None if state is None else state.cpu(), n)
            outs.append(o)
            f0 += n
        out_s = torch.cat(outs, dim=1)
        assert_close(out_s.float().cpu().numpy(), out_all.float().cpu().numpy(), "chunked out")
        assert_close(state.cpu().numpy(), s_all.cpu().numpy(), "chunked state")
    ref, sref = oracle.gla_forward(q, k, v, g, F, s, 1e-6)
    assert_close(out_all.float().cpu().numpy(), ref, "out")
    assert_close(s_all.cpu().numpy(), sref, "state_out")


def test_state_options_and_aliasing():
    F, T, d = 3, 150, 64
    w, q, k, v, g, s = small_case(2, 2, F, T, d, True, seed=9)
    dev = torch.device("cuda")
    qd, kd, vd, gd, sd = (x.to(dev) for x in (q, k, v, g, s))
    B, N, H, _ = q.shape
    out1 = torch.empty_like(qd)
    so1 = torch.empty_like(sd)
    gla().gla_forward(qd, kd, vd, gd, sd, so1, out1, B, H, F, T, d, 1e-6)
    # state_out aliasing state_in (in-place update) gives the same bits
    s_inplace = sd.clone()
    out2 = torch.empty_like(qd)
    gla().gla_forward(qd, kd, vd, gd, s_inplace, s_inplace, out2, B, H, F, T, d, 1e-6)
    # no state_out requested: same output
    out3 = torch.empty_like(qd)
    gla().gla_forward(qd, kd, vd, gd, sd, None, out3, B, H, F, T, d, 1e-6)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2) and torch.equal(out1, out3)
    assert torch.equal(so1, s_inplace)
    # NULL state_in == explicit zeros
    z = torch.zeros_like(sd)
    out4, so4 = torch.empty_like(qd), torch.empty_like(sd)
    out5, so5 = torch.empty_like(qd), torch.empty_like(sd)
    gla().gla_forward(qd, kd, vd, gd, None, so4, out4, B, H, F, T, d, 1e-6)
    gla().gla_forward(qd, kd, vd, gd, z, so5, out5, B, H, F, T, d, 1e-6)
    torch.cuda.synchronize()
    assert torch.equal(out4, out5) and torch.equal(so4, so5)


def test_deterministic():
    F, T, d = 5, 1000, 128
    w, q, k, v, g, s = small_case(2, 4, F, T, d, False, seed=12)
    o1, s1 = run_gpu(q, k, v, g, None, F)
    o2, s2 = run_gpu(q, k, v, g, None, F)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_trim_workspace_between_calls():
    F, T, d = 4, 500, 128
    w, q, k, v, g, s = small_case(2, 4, F, T, d, True, seed=31)
    o1, s1 = run_gpu(q, k, v, g, s, F)
    gla().gla_trim_workspace()
    o2, s2 = run_gpu(q, k, v, g, s, F)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_guard_bands_untouched():
    """Writes stay inside out and state_out (TMA store clipping at ragged
    frame ends, scan bounds)."""
    F, T, d, B, H = 3, 37, 128, 2, 3
    w, q, k, v, g, s = small_case(B, H, F, T, d, True, seed=21)
    dev = torch.device("cuda")
    qd, kd, vd, gd, sd = (x.to(dev) for x in (q, k, v, g, s))
    pad = 64
    n_out = q.numel()
    buf = torch.full((n_out + 2 * pad,), 1234.5, device=dev, dtype=torch.bfloat16)
    out = buf[pad:pad + n_out]
    sbuf = torch.full((s.numel() + 2 * pad,), -777.0, device=dev, dtype=torch.float32)
    so = sbuf[pad:pad + s.numel()]
    gla().gla_forward(qd, kd, vd, gd, sd, so.data_ptr(), out.data_ptr(), B, H, F, T, d, 1e-6)
    torch.cuda.synchronize()
    assert torch.all(buf[:pad] == 1234.5) and torch.all(buf[pad + n_out:] == 1234.5)
    assert torch.all(sbuf[:pad] == -777.0) and torch.all(sbuf[pad + s.numel():] == -777.0)
    ref, sref = oracle.gla_forward(q, k, v, g, F, s, 1e-6)
    assert_close(out.view(q.shape).float().cpu().numpy(), ref, "out")
    assert_close(so.view(s.shape).cpu().numpy(), sref, "state_out")


def test_empty_and_degenerate_sizes():
    dev = torch.device("cuda")
    d, B, H = 64, 2, 3
    s = torch.randn(B, H, d, d + 1, generator=torch.Generator().manual_seed(3)).to(dev)
    # frames = 0: state passes through
    so = torch.empty_like(s)
    e = torch.empty(B, 0, H, d, device=dev, dtype=torch.bfloat16)
    g0 = torch.empty(B, 0, H, device=dev)
    gla().gla_forward(e, e, e, g0, s, so, e, B, H, 0, 128, d, 1e-6)
    torch.cuda.synchronize()
    assert torch.equal(so, s)
    # frames > 0 with no tokens: only the decays act
    g = torch.randn(B, 3, H, generator=torch.Generator().manual_seed(4)).to(dev)
    gla().gla_forward(e, e, e, g, s, so, e, B, H, 3, 0, d, 1e-6)
    torch.cuda.synchronize()
    a = torch.sigmoid(g.double()).prod(dim=1)  # [B, H]
    ref = s.double() * a[:, :, None, None]
    assert_close(so.cpu().numpy(), ref.cpu().numpy(), "decay-only state")
    # B = 0: nothing happens, no error
    gla().gla_forward(None, None, None, None, None, None, None, 0, H, 3, 16, d, 1e-6)


def test_bad_alignment_rejected_on_device_pointers():
    dev = torch.device("cuda")
    q = torch.zeros(1, 32 + 8, 1, 32, device=dev, dtype=torch.bfloat16)
    g = torch.zeros(1, 2, 1, device=dev)
    out = torch.zeros_like(q)
    import gated_linear_attention_frame_b200 as gl

    with pytest.raises(gl.GLAError) as ei:
        gl.gla_forward(q.data_ptr() + 2, q, q, g, None, None, out, 1, 1, 2, 16, 32, 1e-6)
    assert ei.value.status == gl.GLA_ERR_ALIGN


# ------------------------------------------------ full-size layer workloads


def _sampled_heads(w, n):
    r = np.random.default_rng(w.index)
    pairs = [(b, h) for b in range(w.B) for h in range(w.H)]
    idx = r.choice(len(pairs), size=min(n, len(pairs)), replace=False)
    return [pairs[i] for i in sorted(idx)]


@pytest.mark.parametrize("name,nheads", [("480p-5s", 3), ("720p-5s", 3), ("720p-60s", 2)])
def test_full_size_workload_sampled_heads(name, nheads):
    w = WORKLOADS[name]
    dev = torch.device("cuda")
    q, k, v, g = make_inputs(w, device=dev)
    out = torch.empty_like(q)
    so = torch.empty(w.B, w.H, w.d, w.d + 1, device=dev)
    gla().gla_forward(q, k, v, g, None, so, out, w.B, w.H, w.frames, w.tokens_per_frame, w.d,
                      w.eps)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    for b, h in _sampled_heads(w, nheads):
        ref, sref = oracle.gla_head(q[b, :, h].cpu(), k[b, :, h].cpu(), v[b, :, h].cpu(),
                                    g[b, :, h].cpu(), w.tokens_per_frame, None, w.eps)
        assert_close(out[b, :, h].float().cpu().numpy(), ref, "%s out b%d h%d" % (name, b, h))
        assert_close(so[b, h].cpu().numpy(), sref, "%s state b%d h%d" % (name, b, h))


def test_streaming_workload_64_calls():
    """B=8 sequences, one 3680-token frame per call, fp32 state carried over
    64 calls.  The oracle carries its own fp64 state for sampled heads."""
    w = WORKLOADS["stream"]
    dev = torch.device("cuda")
    s0 = make_state(w)
    state = s0.to(dev)
    heads = _sampled_heads(w, 3)
    ref_state = {bh: s0[bh[0], bh[1]].double().numpy() for bh in heads}
    out = torch.empty(w.B, w.tokens, w.H, w.d, device=dev, dtype=torch.bfloat16)
    for call in range(w.calls):
        qd, kd, vd, gd = make_inputs(w, call=call, device=dev)
        gla().gla_forward(qd, kd, vd, gd, state, state, out, w.B, w.H, 1, w.tokens_per_frame,
                          w.d, w.eps)
        check = call % 8 == 0 or call == w.calls - 1
        for (b, h) in heads:
            ref, ref_state[(b, h)] = oracle.gla_head(qd[b, :, h].cpu(), kd[b, :, h].cpu(),
                                                     vd[b, :, h].cpu(), gd[b, :, h].cpu(),
                                                     w.tokens_per_frame, ref_state[(b, h)], w.eps)
            if check:
                assert_close(out[b, :, h].float().cpu().numpy(), ref,
                             "call %d out b%d h%d" % (call, b, h))
    torch.cuda.synchronize()
    for (b, h) in heads:
        assert_close(state[b, h].cpu().numpy(), ref_state[(b, h)], "final state b%d h%d" % (b, h))
