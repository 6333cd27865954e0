"""The C-ABI library: builds, loads without a GPU, exports every function that
include/gla.h declares, and rejects bad arguments before any CUDA call."""

import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gla.h")


@pytest.fixture(scope="module")
def lib():
    from gated_linear_attention_frame_b200.build import build

    build()
    import gated_linear_attention_frame_b200 as g

    return g.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\**\s*(gla_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("gla_forward", "gla_error_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert names
    for n in names:
        assert hasattr(lib, n), n
    import gated_linear_attention_frame_b200 as g

    assert set(names) == set(g.EXPORTED)


def test_error_strings(lib):
    import gated_linear_attention_frame_b200 as g

    seen = set()
    for st in range(0, 10):
        s = g.gla_error_string(st)
        assert s and s != "unknown status"
        seen.add(s)
    assert len(seen) == 10
    assert g.gla_error_string(99) == "unknown status"
    assert g.gla_version() >= 100


def _call(lib, q=None, k=None, v=None, g=None, s_in=None, s_out=None, out=None,
          B=1, H=1, F=1, T=16, d=32, eps=1e-6):
    return lib.gla_forward(q, k, v, g, s_in, s_out, out, B, H, F, T, d, eps, None)


FAKE = 1 << 20  # never dereferenced: validation fails first


def test_validation_before_any_cuda_call(lib):
    import gated_linear_attention_frame_b200 as gl

    ok = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, out=FAKE)
    assert _call(lib, d=48, **ok) == gl.GLA_ERR_UNSUPPORTED_D
    assert _call(lib, d=256, **ok) == gl.GLA_ERR_UNSUPPORTED_D
    assert _call(lib, B=-1, **ok) == gl.GLA_ERR_SHAPE
    assert _call(lib, T=-5, **ok) == gl.GLA_ERR_SHAPE
    assert _call(lib, F=1 << 20, T=1 << 12, **ok) == gl.GLA_ERR_SHAPE
    assert _call(lib, **dict(ok, q=None)) == gl.GLA_ERR_NULL
    assert _call(lib, **dict(ok, out=None)) == gl.GLA_ERR_NULL
    assert _call(lib, **dict(ok, g=None)) == gl.GLA_ERR_NULL
    assert _call(lib, **dict(ok, v=FAKE + 8)) == gl.GLA_ERR_ALIGN
    assert _call(lib, **dict(ok, out=FAKE + 2)) == gl.GLA_ERR_ALIGN
    assert _call(lib, **dict(ok, s_in=FAKE + 2)) == gl.GLA_ERR_ALIGN
    # empty batch or heads: nothing to do, no device needed
    assert _call(lib, B=0, **ok) == gl.GLA_OK
    assert _call(lib, H=0) == gl.GLA_OK


def _bcall(lib, d=128, B=1, H=1, F=1, T=16, **kw):
    p = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, s_in=None, dout=FAKE, ds_out=None, dq=FAKE,
             dk=FAKE, dv=FAKE, dg=FAKE, ds_in=None)
    p.update(kw)
    return lib.gla_backward(p["q"], p["k"], p["v"], p["g"], p["s_in"], p["dout"], p["ds_out"],
                            p["dq"], p["dk"], p["dv"], p["dg"], p["ds_in"], B, H, F, T, d, 1e-6,
                            None)


def test_backward_validation_before_any_cuda_call(lib):
    import gated_linear_attention_frame_b200 as gl

    assert _bcall(lib, d=64) == gl.GLA_ERR_UNSUPPORTED_D   # backward is built for d = 128
    assert _bcall(lib, d=32) == gl.GLA_ERR_UNSUPPORTED_D
    assert _bcall(lib, B=-1) == gl.GLA_ERR_SHAPE
    for name in ("q", "k", "v", "dout", "dq", "dk", "dv", "dg", "g"):
        assert _bcall(lib, **{name: None}) == gl.GLA_ERR_NULL, name
    for name in ("q", "dout", "dq", "dk", "dv"):
        assert _bcall(lib, **{name: FAKE + 8}) == gl.GLA_ERR_ALIGN, name
    for name in ("dg", "ds_in", "ds_out", "s_in"):
        assert _bcall(lib, **{name: FAKE + 2}) == gl.GLA_ERR_ALIGN, name
    # no tokens: dq/dk/dv/dout may be NULL; no frames: dgate_logits may be NULL
    assert _bcall(lib, B=0) == gl.GLA_OK
    assert _bcall(lib, H=0, dg=None, dq=None) == gl.GLA_OK
    st = lib.gla_backward_timed(FAKE, FAKE, FAKE, FAKE, None, FAKE, None, FAKE, FAKE, FAKE, FAKE,
                                None, 1, 1, 1, 16, 128, 1e-6, None, None)
    assert st == gl.GLA_ERR_NULL


def test_rope_validation_before_any_cuda_call(lib):
    import ctypes

    import gated_linear_attention_frame_b200 as gl

    def call(rope, d=128, **kw):
        p = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, out=FAKE)
        p.update(kw)
        return lib.gla_forward_rope(p["q"], p["k"], p["v"], p["g"], None, None, p["out"], 1, 1,
                                    1, 16, d, 1e-6,
                                    None if rope is None else ctypes.byref(rope), None)

    assert call(None) == gl.GLA_ERR_NULL
    bad = [gl.rope_config(80, (32, 48, 40)),         # blocks do not sum to d
           gl.rope_config(80, (36, 44, 48)),         # not multiples of 8
           gl.rope_config(80, (-8, 88, 48)),
           gl.rope_config(0, (32, 48, 48)),          # grid_w < 1
           gl.rope_config(80, (32, 48, 48), frame_offset=-1),
           gl.rope_config(80, (32, 48, 48), theta=0.0),
           gl.rope_config(80, (32, 48, 48), theta=float("inf")),
           gl.rope_config(80, (32, 48, 48), theta=float("nan"))]
    for r in bad:
        assert call(r) == gl.GLA_ERR_ROPE, (r.grid_w, r.dim_t, r.dim_y, r.dim_x, r.theta)
    assert call(gl.rope_config(8, (8, 8, 16)), d=32, q=None) == gl.GLA_ERR_NULL
    assert call(gl.rope_config(8, (32, 48, 48)), d=48) == gl.GLA_ERR_UNSUPPORTED_D
    # valid configuration, empty batch: nothing to do
    assert lib.gla_forward_rope(FAKE, FAKE, FAKE, FAKE, None, None, FAKE, 0, 1, 1, 16, 128, 1e-6,
                                ctypes.byref(gl.rope_config(80)), None) == gl.GLA_OK


def test_gdn_validation_before_any_cuda_call(lib):
    import gated_linear_attention_frame_b200 as gl

    def call(beta=FAKE, d=128, B=1, **kw):
        p = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, out=FAKE)
        p.update(kw)
        return lib.gla_forward_gdn(p["q"], p["k"], p["v"], p["g"], beta, None, None, p["out"], B,
                                   1, 1, 16, d, 1e-6, None)

    assert call(beta=None) == gl.GLA_ERR_NULL
    assert call(beta=FAKE + 2) == gl.GLA_ERR_ALIGN
    assert call(d=48) == gl.GLA_ERR_UNSUPPORTED_D
    assert call(g=None) == gl.GLA_ERR_NULL
    assert call(B=0) == gl.GLA_OK
    assert lib.gla_forward_gdn_timed(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, 1, 1, 1, 16,
                                     128, 1e-6, None, None) == gl.GLA_ERR_NULL


def test_softmax_anchor_validation_before_any_cuda_call(lib):
    import gated_linear_attention_frame_b200 as gl

    def call(d=128, W=2, S=0, q=FAKE, out=FAKE, z=None, B=1):
        return lib.gla_softmax_anchor(q, FAKE, FAKE, z, out, B, 1, 2, 16, d, W, S, None)

    assert call(d=64) == gl.GLA_ERR_UNSUPPORTED_D
    assert call(W=0) == gl.GLA_ERR_SHAPE
    assert call(S=-1) == gl.GLA_ERR_SHAPE
    assert call(q=None) == gl.GLA_ERR_NULL
    assert call(out=FAKE + 8) == gl.GLA_ERR_ALIGN
    assert call(z=FAKE + 8) == gl.GLA_ERR_ALIGN
    assert call(B=0) == gl.GLA_OK
    assert lib.gla_softmax_anchor_timed(FAKE, FAKE, FAKE, None, FAKE, 1, 1, 2, 16, 128, 2, 0, None,
                                        None) == gl.GLA_ERR_NULL


def test_timed_variant_requires_events(lib):
    import gated_linear_attention_frame_b200 as gl

    st = lib.gla_forward_timed(FAKE, FAKE, FAKE, FAKE, None, None, FAKE, 1, 1, 1, 16, 32, 1e-6,
                               None, None)
    assert st == gl.GLA_ERR_NULL


def test_device_fault_rejects_null(lib):
    import gated_linear_attention_frame_b200 as gl

    assert lib.gla_device_fault(None, None) == gl.GLA_ERR_NULL


def test_binding_marshalling_errors():
    import torch

    import gated_linear_attention_frame_b200 as gl

    q = torch.zeros(1, 16, 1, 32, dtype=torch.float32)
    with pytest.raises(TypeError):
        gl.gla_forward(q, q, q, None, None, None, q, 1, 1, 1, 16, 32, 1e-6, 0)
    qb = torch.zeros(1, 16, 1, 32, dtype=torch.bfloat16)  # CPU tensor: not a device pointer
    g = torch.zeros(1, 1, 1)
    with pytest.raises(ValueError):
        gl.gla_forward(qb, qb, qb, g, None, None, qb, 1, 1, 1, 16, 32, 1e-6, 0)


def test_missing_library_fails_loudly(tmp_path):
    from gated_linear_attention_frame_b200._binding import load_library

    with pytest.raises(ImportError):
        load_library(str(tmp_path / "libgla.so"))


def test_alloc_failure_hook_is_host_only(lib):
    # arming and disarming the hook makes no CUDA call (this runs without a GPU)
    assert lib.gla_inject_alloc_failure(3) == 0
    assert lib.gla_inject_alloc_failure(0) == 0


def test_anchor_step_validation_before_any_cuda_call(lib):
    # d != 128, negative frame, missing caches: rejected without touching CUDA
    vp = FAKE
    assert lib.gla_softmax_anchor_step(vp, vp, vp, None, vp, vp, vp, vp, vp, 1, 1, 64, 64, 1, 2,
                                       64, None) == 4
    assert lib.gla_softmax_anchor_step(vp, vp, vp, None, vp, vp, vp, vp, vp, 1, 1, 64, 128, -1,
                                       2, 64, None) == 3
    assert lib.gla_softmax_anchor_step(vp, vp, vp, None, vp, vp, None, None, vp, 1, 1, 64, 128, 3,
                                       2, 64, None) == 1


def test_saved_context_calls_validate_before_any_cuda_call(lib):
    # gla_forward_train / gla_backward_saved: d != 128, a missing or
    # misaligned context are rejected without touching CUDA
    vp = FAKE
    odd = FAKE + 16  # 16-byte but not 256-byte aligned
    assert lib.gla_saved_bytes(2, 24, 21, 3680, 128) == 133152768
    assert lib.gla_saved_bytes(2, 24, 21, 3680, 64) == 0
    assert lib.gla_saved_bytes(-1, 24, 21, 3680, 128) == 0
    # forward_train: q, k, v, g, state_in, state_out, out, saved, B, H, F, T, d, eps, stream
    assert lib.gla_forward_train(vp, vp, vp, vp, None, None, vp, vp, 1, 1, 1, 64, 64, 1e-6,
                                 None) == 4
    assert lib.gla_forward_train(vp, vp, vp, vp, None, None, vp, None, 1, 1, 1, 64, 128, 1e-6,
                                 None) == 1
    assert lib.gla_forward_train(vp, vp, vp, vp, None, None, vp, odd, 1, 1, 1, 64, 128, 1e-6,
                                 None) == 2
    # backward_saved: q, k, v, g, state_in, saved, dout, dstate_out, dq, dk, dv, dg, dstate_in, ...
    assert lib.gla_backward_saved(vp, vp, vp, vp, None, vp, vp, None, vp, vp, vp, vp, None, 1, 1,
                                  1, 64, 64, 1e-6, None) == 4
    assert lib.gla_backward_saved(vp, vp, vp, vp, None, None, vp, None, vp, vp, vp, vp, None, 1,
                                  1, 1, 64, 128, 1e-6, None) == 1
    assert lib.gla_backward_saved(vp, vp, vp, vp, None, odd, vp, None, vp, vp, vp, vp, None, 1, 1,
                                  1, 64, 128, 1e-6, None) == 2
