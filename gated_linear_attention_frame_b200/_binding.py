"""ctypes binding of libgla.so, with the same names as the C ABI (include/gla.h).

Only argument marshalling happens here: tensors become device pointers and
the stream becomes a raw cudaStream_t; every step of the computation runs in
the library's CUDA kernels.  If the shared library is missing or cannot be
loaded, importing the package raises -- there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgla.so")

GLA_OK = 0
GLA_ERR_NULL = 1
GLA_ERR_ALIGN = 2
GLA_ERR_SHAPE = 3
GLA_ERR_UNSUPPORTED_D = 4
GLA_ERR_ALLOC = 5
GLA_ERR_LAUNCH = 6
GLA_ERR_DEVICE = 7
GLA_ERR_SCRATCH = 8
GLA_ERR_ROPE = 9

EXPORTED = ("gla_forward", "gla_forward_timed", "gla_forward_noalloc", "gla_noalloc_scratch_bytes",
            "gla_forward_rope", "gla_forward_rope_timed", "gla_forward_gdn", "gla_forward_gdn_timed",
            "gla_softmax_anchor", "gla_softmax_anchor_timed", "gla_softmax_anchor_step",
            "gla_backward", "gla_backward_timed", "gla_saved_bytes", "gla_forward_train",
            "gla_backward_saved", "gla_backward_saved_timed",
            "gla_trim_workspace", "gla_set_workspace_retention", "gla_inject_alloc_failure",
            "gla_set_wait_limit_ns", "gla_inject_stall", "gla_error_string", "gla_device_fault",
            "gla_version")


class RopeConfig(ctypes.Structure):
    """gla_rope_config of include/gla.h (3D rotary position embedding)."""

    _fields_ = [("grid_w", ctypes.c_int), ("frame_offset", ctypes.c_int),
                ("dim_t", ctypes.c_int), ("dim_y", ctypes.c_int), ("dim_x", ctypes.c_int),
                ("theta", ctypes.c_float)]


def rope_config(grid_w: int, dims=(32, 48, 48), frame_offset: int = 0,
                theta: float = 10000.0) -> RopeConfig:
    return RopeConfig(int(grid_w), int(frame_offset), int(dims[0]), int(dims[1]), int(dims[2]),
                      float(theta))


class GLAError(RuntimeError):
    def __init__(self, status: int, where: str = "gla_forward"):
        self.status = int(status)
        super().__init__("%s failed: %s (status %d)" % (where, gla_error_string(status), status))


_lib = None


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load libgla.so (once) and declare the C signatures."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(
            "libgla.so not found at %s; build it with "
            "`python -m gated_linear_attention_frame_b200.build`" % p)
    lib = ctypes.CDLL(p)
    vp, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    fwd = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, vp]
    lib.gla_forward.argtypes = fwd
    lib.gla_forward.restype = i32
    lib.gla_forward_timed.argtypes = fwd + [ctypes.POINTER(vp)]
    lib.gla_forward_timed.restype = i32
    lib.gla_forward_noalloc.argtypes = fwd
    lib.gla_forward_noalloc.restype = i32
    anc = [vp] * 5 + [i32] * 7 + [vp]
    lib.gla_softmax_anchor.argtypes = anc
    lib.gla_softmax_anchor.restype = i32
    lib.gla_softmax_anchor_timed.argtypes = anc + [ctypes.POINTER(vp)]
    lib.gla_softmax_anchor_timed.restype = i32
    lib.gla_softmax_anchor_step.argtypes = [vp] * 9 + [i32] * 7 + [vp]
    lib.gla_softmax_anchor_step.restype = i32
    gdn = fwd[:4] + [vp] + fwd[4:]
    lib.gla_forward_gdn.argtypes = gdn
    lib.gla_forward_gdn.restype = i32
    lib.gla_forward_gdn_timed.argtypes = gdn + [ctypes.POINTER(vp)]
    lib.gla_forward_gdn_timed.restype = i32
    rope_p = ctypes.POINTER(RopeConfig)
    lib.gla_forward_rope.argtypes = fwd[:13] + [rope_p, vp]
    lib.gla_forward_rope.restype = i32
    lib.gla_forward_rope_timed.argtypes = fwd[:13] + [rope_p, vp, ctypes.POINTER(vp)]
    lib.gla_forward_rope_timed.restype = i32
    bwd = [vp] * 12 + [i32, i32, i32, i32, i32, f32, vp]
    lib.gla_backward.argtypes = bwd
    lib.gla_backward.restype = i32
    lib.gla_backward_timed.argtypes = bwd + [ctypes.POINTER(vp)]
    lib.gla_backward_timed.restype = i32
    lib.gla_saved_bytes.argtypes = [i32] * 5
    lib.gla_saved_bytes.restype = ctypes.c_size_t
    lib.gla_forward_train.argtypes = [vp] * 8 + [i32] * 5 + [f32, vp]
    lib.gla_forward_train.restype = i32
    bwds = [vp] * 13 + [i32, i32, i32, i32, i32, f32, vp]  # gla_backward's + saved
    lib.gla_backward_saved.argtypes = bwds
    lib.gla_backward_saved.restype = i32
    lib.gla_backward_saved_timed.argtypes = bwds + [ctypes.POINTER(vp)]
    lib.gla_backward_saved_timed.restype = i32
    lib.gla_noalloc_scratch_bytes.argtypes = []
    lib.gla_noalloc_scratch_bytes.restype = ctypes.c_size_t
    lib.gla_trim_workspace.argtypes = []
    lib.gla_trim_workspace.restype = i32
    lib.gla_set_workspace_retention.argtypes = [ctypes.c_ulonglong]
    lib.gla_set_workspace_retention.restype = i32
    lib.gla_inject_alloc_failure.argtypes = [i32]
    lib.gla_inject_alloc_failure.restype = i32
    lib.gla_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    lib.gla_set_wait_limit_ns.restype = i32
    lib.gla_inject_stall.argtypes = [ctypes.c_longlong]
    lib.gla_inject_stall.restype = i32
    lib.gla_error_string.argtypes = [i32]
    lib.gla_error_string.restype = ctypes.c_char_p
    lib.gla_device_fault.argtypes = [vp, ctypes.POINTER(ctypes.c_uint)]
    lib.gla_device_fault.restype = i32
    lib.gla_version.argtypes = []
    lib.gla_version.restype = i32
    if path is None:
        _lib = lib
    return lib


def _ptr(x) -> int | None:
    """Device pointer of a CUDA tensor, an int address, or None (-> NULL)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, torch.Tensor):
        if x.numel() == 0:
            return x.data_ptr() or None
        if not x.is_cuda:
            raise ValueError("gla: tensors must be on a CUDA device (got %s)" % x.device)
        if not x.is_contiguous():
            raise ValueError("gla: tensors must be contiguous")
        return x.data_ptr()
    raise TypeError("gla: expected a torch.Tensor, an int address or None, got %r" % type(x))


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check_dtypes(q, k, v, gate_logits, state_in, state_out, out):
    for name, t, dt in (("q", q, torch.bfloat16), ("k", k, torch.bfloat16),
                        ("v", v, torch.bfloat16), ("out", out, torch.bfloat16),
                        ("gate_logits", gate_logits, torch.float32),
                        ("state_in", state_in, torch.float32),
                        ("state_out", state_out, torch.float32)):
        if isinstance(t, torch.Tensor) and t.dtype != dt:
            raise TypeError("gla: %s must be %s, got %s" % (name, dt, t.dtype))


def gla_forward(q, k, v, gate_logits, state_in, state_out, out, B, H, frames,
                tokens_per_frame, d, eps, stream=None) -> None:
    """Enqueue one layer call (see include/gla.h).  Tensors or raw device
    addresses; raises GLAError on a nonzero status."""
    _check_dtypes(q, k, v, gate_logits, state_in, state_out, out)
    lib = load_library()
    st = lib.gla_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_logits), _ptr(state_in),
                         _ptr(state_out), _ptr(out), int(B), int(H), int(frames),
                         int(tokens_per_frame), int(d), float(eps), _stream(stream))
    if st != GLA_OK:
        raise GLAError(st)


def gla_forward_timed(q, k, v, gate_logits, state_in, state_out, out, B, H, frames,
                      tokens_per_frame, d, eps, stream, events) -> None:
    """gla_forward that records 4 CUDA events around the three kernels
    (`events`: 4 torch.cuda.Event(enable_timing=True))."""
    _check_dtypes(q, k, v, gate_logits, state_in, state_out, out)
    lib = load_library()
    for e in events:
        if e.cuda_event == 0:  # torch creates the CUDA event at its first record
            e.record()
    arr = (ctypes.c_void_p * 4)(*[e.cuda_event for e in events])
    st = lib.gla_forward_timed(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_logits), _ptr(state_in),
                               _ptr(state_out), _ptr(out), int(B), int(H), int(frames),
                               int(tokens_per_frame), int(d), float(eps), _stream(stream),
                               ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p)))
    if st != GLA_OK:
        raise GLAError(st, "gla_forward_timed")


def gla_forward_noalloc(q, k, v, gate_logits, state_in, state_out, out, B, H, frames,
                        tokens_per_frame, d, eps, stream=None) -> None:
    """gla_forward with its workspace in the library's fixed device scratch
    array instead of a fresh allocation (see include/gla.h).  For callers
    that must not allocate device memory; problems whose workspace exceeds
    gla_noalloc_scratch_bytes() raise GLAError(GLA_ERR_SCRATCH)."""
    _check_dtypes(q, k, v, gate_logits, state_in, state_out, out)
    lib = load_library()
    st = lib.gla_forward_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_logits), _ptr(state_in),
                                 _ptr(state_out), _ptr(out), int(B), int(H), int(frames),
                                 int(tokens_per_frame), int(d), float(eps), _stream(stream))
    if st != GLA_OK:
        raise GLAError(st, "gla_forward_noalloc")


def gla_softmax_anchor(q, k, v, gate_z, out, B, H, frames, tokens_per_frame, d, window_frames,
                       n_sink, stream=None) -> None:
    """The softmax anchor layer: attention sinks + a local window of frames,
    optional sigmoid output gate (see include/gla.h; d = 128)."""
    for name, t in (("q", q), ("k", k), ("v", v), ("gate_z", gate_z), ("out", out)):
        if isinstance(t, torch.Tensor) and t.dtype != torch.bfloat16:
            raise TypeError("gla: %s must be torch.bfloat16, got %s" % (name, t.dtype))
    st = load_library().gla_softmax_anchor(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_z), _ptr(out),
                                           int(B), int(H), int(frames), int(tokens_per_frame),
                                           int(d), int(window_frames), int(n_sink),
                                           _stream(stream))
    if st != GLA_OK:
        raise GLAError(st, "gla_softmax_anchor")


def gla_softmax_anchor_timed(q, k, v, gate_z, out, B, H, frames, tokens_per_frame, d,
                             window_frames, n_sink, stream, events) -> None:
    """gla_softmax_anchor with 2 CUDA events around the kernel."""
    lib = load_library()
    for e in events:
        if e.cuda_event == 0:
            e.record()
    arr = (ctypes.c_void_p * 2)(*[e.cuda_event for e in events])
    st = lib.gla_softmax_anchor_timed(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_z), _ptr(out), int(B),
                                      int(H), int(frames), int(tokens_per_frame), int(d),
                                      int(window_frames), int(n_sink), _stream(stream),
                                      ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p)))
    if st != GLA_OK:
        raise GLAError(st, "gla_softmax_anchor_timed")


def softmax_anchor(q, k, v, frames, window_frames, n_sink=0, gate_z=None, out=None, stream=None):
    """Convenience wrapper of gla_softmax_anchor; returns out."""
    B, N, H, d = q.shape
    T = N // frames if frames else 0
    if frames and N % frames:
        raise ValueError("token axis %d is not a multiple of frames %d" % (N, frames))
    if out is None:
        out = torch.empty_like(q)
    gla_softmax_anchor(q, k, v, gate_z, out, B, H, frames, T, d, window_frames, n_sink, stream)
    return out


def gla_softmax_anchor_step(q, k, v, gate_z, sink_k, sink_v, win_k, win_v, out, B, H,
                            tokens_per_frame, d, frame, window_frames, n_sink,
                            stream=None) -> None:
    """The softmax anchor layer for one new frame of a rollout, from the sink
    and window caches (see include/gla.h; d = 128)."""
    for name, t in (("q", q), ("k", k), ("v", v), ("gate_z", gate_z), ("sink_k", sink_k),
                    ("sink_v", sink_v), ("win_k", win_k), ("win_v", win_v), ("out", out)):
        if isinstance(t, torch.Tensor) and t.dtype != torch.bfloat16:
            raise TypeError("gla: %s must be torch.bfloat16, got %s" % (name, t.dtype))
    st = load_library().gla_softmax_anchor_step(
        _ptr(q), _ptr(k), _ptr(v), _ptr(gate_z), _ptr(sink_k), _ptr(sink_v), _ptr(win_k),
        _ptr(win_v), _ptr(out), int(B), int(H), int(tokens_per_frame), int(d), int(frame),
        int(window_frames), int(n_sink), _stream(stream))
    if st != GLA_OK:
        raise GLAError(st, "gla_softmax_anchor_step")


def softmax_anchor_step(q, k, v, frame, window_frames, n_sink=0, sink_k=None, sink_v=None,
                        win_k=None, win_v=None, gate_z=None, out=None, stream=None):
    """Convenience wrapper of gla_softmax_anchor_step: q, k, v [B, T, H, d] of
    frame `frame`; returns out."""
    B, T, H, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    gla_softmax_anchor_step(q, k, v, gate_z, sink_k, sink_v, win_k, win_v, out, B, H, T, d,
                            frame, window_frames, n_sink, stream)
    return out


def gla_forward_gdn(q, k, v, gate_logits, beta_logits, state_in, state_out, out, B, H, frames,
                    tokens_per_frame, d, eps, stream=None) -> None:
    """The frame-wise gated delta-rule variant (see include/gla.h)."""
    _check_dtypes(q, k, v, gate_logits, state_in, state_out, out)
    _check_dtypes(None, None, None, beta_logits, None, None, None)
    lib = load_library()
    st = lib.gla_forward_gdn(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_logits), _ptr(beta_logits),
                             _ptr(state_in), _ptr(state_out), _ptr(out), int(B), int(H),
                             int(frames), int(tokens_per_frame), int(d), float(eps),
                             _stream(stream))
    if st != GLA_OK:
        raise GLAError(st, "gla_forward_gdn")


def gla_forward_gdn_timed(q, k, v, gate_logits, beta_logits, state_in, state_out, out, B, H,
                          frames, tokens_per_frame, d, eps, stream, events) -> None:
    """gla_forward_gdn that records 4 CUDA events around the kernels."""
    _check_dtypes(q, k, v, gate_logits, state_in, state_out, out)
    lib = load_library()
    for e in events:
        if e.cuda_event == 0:
            e.record()
    arr = (ctypes.c_void_p * 4)(*[e.cuda_event for e in events])
    st = lib.gla_forward_gdn_timed(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_logits),
                                   _ptr(beta_logits), _ptr(state_in), _ptr(state_out), _ptr(out),
                                   int(B), int(H), int(frames), int(tokens_per_frame), int(d),
                                   float(eps), _stream(stream),
                                   ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p)))
    if st != GLA_OK:
        raise GLAError(st, "gla_forward_gdn_timed")


def gla_forward_rope(q, k, v, gate_logits, state_in, state_out, out, B, H, frames,
                     tokens_per_frame, d, eps, rope: RopeConfig, stream=None) -> None:
    """gla_forward with the 3D rotary position embedding (see include/gla.h)."""
    _check_dtypes(q, k, v, gate_logits, state_in, state_out, out)
    lib = load_library()
    st = lib.gla_forward_rope(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_logits), _ptr(state_in),
                              _ptr(state_out), _ptr(out), int(B), int(H), int(frames),
                              int(tokens_per_frame), int(d), float(eps),
                              None if rope is None else ctypes.byref(rope), _stream(stream))
    if st != GLA_OK:
        raise GLAError(st, "gla_forward_rope")


def gla_forward_rope_timed(q, k, v, gate_logits, state_in, state_out, out, B, H, frames,
                           tokens_per_frame, d, eps, rope: RopeConfig, stream, events) -> None:
    """gla_forward_rope that records 4 CUDA events around the kernels."""
    _check_dtypes(q, k, v, gate_logits, state_in, state_out, out)
    lib = load_library()
    for e in events:
        if e.cuda_event == 0:
            e.record()
    arr = (ctypes.c_void_p * 4)(*[e.cuda_event for e in events])
    st = lib.gla_forward_rope_timed(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_logits),
                                    _ptr(state_in), _ptr(state_out), _ptr(out), int(B), int(H),
                                    int(frames), int(tokens_per_frame), int(d), float(eps),
                                    ctypes.byref(rope), _stream(stream),
                                    ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p)))
    if st != GLA_OK:
        raise GLAError(st, "gla_forward_rope_timed")


def _check_bwd_dtypes(dout, dstate_out, dq, dk, dv, dgate_logits, dstate_in):
    for name, t, dt in (("dout", dout, torch.bfloat16), ("dq", dq, torch.bfloat16),
                        ("dk", dk, torch.bfloat16), ("dv", dv, torch.bfloat16),
                        ("dstate_out", dstate_out, torch.float32),
                        ("dgate_logits", dgate_logits, torch.float32),
                        ("dstate_in", dstate_in, torch.float32)):
        if isinstance(t, torch.Tensor) and t.dtype != dt:
            raise TypeError("gla: %s must be %s, got %s" % (name, dt, t.dtype))


def _bwd_args(q, k, v, gate_logits, state_in, dout, dstate_out, dq, dk, dv, dgate_logits,
              dstate_in, B, H, frames, tokens_per_frame, d, eps, stream):
    _check_dtypes(q, k, v, gate_logits, state_in, None, dq)
    _check_bwd_dtypes(dout, dstate_out, dq, dk, dv, dgate_logits, dstate_in)
    return (_ptr(q), _ptr(k), _ptr(v), _ptr(gate_logits), _ptr(state_in), _ptr(dout),
            _ptr(dstate_out), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dgate_logits), _ptr(dstate_in),
            int(B), int(H), int(frames), int(tokens_per_frame), int(d), float(eps),
            _stream(stream))


def gla_backward(q, k, v, gate_logits, state_in, dout, dstate_out, dq, dk, dv, dgate_logits,
                 dstate_in, B, H, frames, tokens_per_frame, d, eps, stream=None) -> None:
    """Enqueue the gradients of one layer call (see include/gla.h; d = 128).
    Tensors or raw device addresses; raises GLAError on a nonzero status."""
    args = _bwd_args(q, k, v, gate_logits, state_in, dout, dstate_out, dq, dk, dv, dgate_logits,
                     dstate_in, B, H, frames, tokens_per_frame, d, eps, stream)
    st = load_library().gla_backward(*args)
    if st != GLA_OK:
        raise GLAError(st, "gla_backward")


def gla_backward_timed(q, k, v, gate_logits, state_in, dout, dstate_out, dq, dk, dv,
                       dgate_logits, dstate_in, B, H, frames, tokens_per_frame, d, eps, stream,
                       events) -> None:
    """gla_backward that records 7 CUDA events around its six kernels
    (`events`: 7 torch.cuda.Event(enable_timing=True))."""
    args = _bwd_args(q, k, v, gate_logits, state_in, dout, dstate_out, dq, dk, dv, dgate_logits,
                     dstate_in, B, H, frames, tokens_per_frame, d, eps, stream)
    lib = load_library()
    for e in events:
        if e.cuda_event == 0:
            e.record()
    arr = (ctypes.c_void_p * 7)(*[e.cuda_event for e in events])
    st = lib.gla_backward_timed(*args, ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p)))
    if st != GLA_OK:
        raise GLAError(st, "gla_backward_timed")


def gla_saved_bytes(B, H, frames, tokens_per_frame, d) -> int:
    """Bytes of the context gla_forward_train saves (0 if d != 128)."""
    return int(load_library().gla_saved_bytes(int(B), int(H), int(frames), int(tokens_per_frame),
                                              int(d)))


def gla_forward_train(q, k, v, gate_logits, state_in, state_out, out, saved, B, H, frames,
                      tokens_per_frame, d, eps, stream=None) -> None:
    """gla_forward that also writes the backward's context into `saved`
    (gla_saved_bytes bytes, 256-byte aligned; see include/gla.h)."""
    st = load_library().gla_forward_train(
        _ptr(q), _ptr(k), _ptr(v), _ptr(gate_logits), _ptr(state_in), _ptr(state_out), _ptr(out),
        _ptr(saved), int(B), int(H), int(frames), int(tokens_per_frame), int(d), float(eps),
        _stream(stream))
    if st != GLA_OK:
        raise GLAError(st, "gla_forward_train")


def _saved_args(args, saved):
    return args[:5] + (_ptr(saved),) + args[5:]


def gla_backward_saved(q, k, v, gate_logits, state_in, saved, dout, dstate_out, dq, dk, dv,
                       dgate_logits, dstate_in, B, H, frames, tokens_per_frame, d, eps,
                       stream=None) -> None:
    """gla_backward from a context of gla_forward_train (no recompute)."""
    args = _bwd_args(q, k, v, gate_logits, state_in, dout, dstate_out, dq, dk, dv, dgate_logits,
                     dstate_in, B, H, frames, tokens_per_frame, d, eps, stream)
    st = load_library().gla_backward_saved(*_saved_args(args, saved))
    if st != GLA_OK:
        raise GLAError(st, "gla_backward_saved")


def gla_backward_saved_timed(q, k, v, gate_logits, state_in, saved, dout, dstate_out, dq, dk, dv,
                             dgate_logits, dstate_in, B, H, frames, tokens_per_frame, d, eps,
                             stream, events) -> None:
    """gla_backward_saved that records 7 CUDA events (as gla_backward_timed)."""
    args = _bwd_args(q, k, v, gate_logits, state_in, dout, dstate_out, dq, dk, dv, dgate_logits,
                     dstate_in, B, H, frames, tokens_per_frame, d, eps, stream)
    lib = load_library()
    for e in events:
        if e.cuda_event == 0:
            e.record()
    arr = (ctypes.c_void_p * 7)(*[e.cuda_event for e in events])
    st = lib.gla_backward_saved_timed(*_saved_args(args, saved),
                                      ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p)))
    if st != GLA_OK:
        raise GLAError(st, "gla_backward_saved_timed")


def gla_noalloc_scratch_bytes() -> int:
    return int(load_library().gla_noalloc_scratch_bytes())


def gla_trim_workspace() -> None:
    """Release the current device's unused workspace memory held by the
    library's pool."""
    st = load_library().gla_trim_workspace()
    if st != GLA_OK:
        raise GLAError(st, "gla_trim_workspace")


def gla_set_workspace_retention(nbytes: int) -> None:
    """Bytes of freed workspace the current device's pool keeps mapped
    between calls (default: all of it; 0 returns everything at each
    synchronisation)."""
    st = load_library().gla_set_workspace_retention(int(nbytes))
    if st != GLA_OK:
        raise GLAError(st, "gla_set_workspace_retention")


def gla_inject_alloc_failure(count: int) -> None:
    """Testing hook: the next `count` workspace allocations fail (GLA_ERR_ALLOC)."""
    load_library().gla_inject_alloc_failure(int(count))


def gla_set_wait_limit_ns(ns: int) -> None:
    """Testing hook: the kernels' barrier-wait limit on the current device
    (0 restores the default of one second)."""
    st = load_library().gla_set_wait_limit_ns(int(ns))
    if st != GLA_OK:
        raise GLAError(st, "gla_set_wait_limit_ns")


def gla_inject_stall(tile: int) -> None:
    """Testing hook: the next state-increment launch withholds one tile on its
    first CTA, so that a wait runs out (see include/gla.h)."""
    st = load_library().gla_inject_stall(int(tile))
    if st != GLA_OK:
        raise GLAError(st, "gla_inject_stall")


def gla_error_string(status: int) -> str:
    return load_library().gla_error_string(int(status)).decode()


def gla_device_fault(stream=None) -> int:
    """Synchronise `stream`, then read and clear the device fault word."""
    code = ctypes.c_uint(0)
    st = load_library().gla_device_fault(_stream(stream), ctypes.byref(code))
    if st != GLA_OK:
        raise GLAError(st, "gla_device_fault")
    return code.value


def gla_version() -> int:
    return load_library().gla_version()


def forward(q, k, v, gate_logits, state_in=None, eps: float = 1e-6, out=None, state_out=None,
            stream=None):
    """Convenience wrapper: shapes from q [B, N, H, d] and gate_logits
    [B, frames, H]; allocates `out` and `state_out` if not given.  Returns
    (out, state_out)."""
    B, N, H, d = q.shape
    frames = gate_logits.shape[1]
    if frames == 0:
        T = 0
    else:
        if N % frames:
            raise ValueError("token axis %d is not a multiple of frames %d" % (N, frames))
        T = N // frames
    if out is None:
        out = torch.empty_like(q)
    if state_out is None:
        state_out = torch.empty(B, H, d, d + 1, device=q.device, dtype=torch.float32)
    gla_forward(q, k, v, gate_logits, state_in, state_out, out, B, H, frames, T, d, eps, stream)
    return out, state_out


def forward_gdn(q, k, v, gate_logits, beta_logits, state_in=None, eps: float = 1e-6, out=None,
                state_out=None, stream=None):
    """Convenience wrapper of gla_forward_gdn; returns (out, state_out)."""
    B, N, H, d = q.shape
    frames = gate_logits.shape[1]
    T = N // frames if frames else 0
    if frames and N % frames:
        raise ValueError("token axis %d is not a multiple of frames %d" % (N, frames))
    if out is None:
        out = torch.empty_like(q)
    if state_out is None:
        state_out = torch.empty(B, H, d, d + 1, device=q.device, dtype=torch.float32)
    gla_forward_gdn(q, k, v, gate_logits, beta_logits, state_in, state_out, out, B, H, frames, T,
                    d, eps, stream)
    return out, state_out


def forward_rope(q, k, v, gate_logits, rope: RopeConfig, state_in=None, eps: float = 1e-6,
                 out=None, state_out=None, stream=None):
    """Convenience wrapper of gla_forward_rope; returns (out, state_out)."""
    B, N, H, d = q.shape
    frames = gate_logits.shape[1]
    T = N // frames if frames else 0
    if frames and N % frames:
        raise ValueError("token axis %d is not a multiple of frames %d" % (N, frames))
    if out is None:
        out = torch.empty_like(q)
    if state_out is None:
        state_out = torch.empty(B, H, d, d + 1, device=q.device, dtype=torch.float32)
    gla_forward_rope(q, k, v, gate_logits, state_in, state_out, out, B, H, frames, T, d, eps,
                     rope, stream)
    return out, state_out


def forward_train(q, k, v, gate_logits, state_in=None, eps: float = 1e-6, out=None,
                  state_out=None, saved=None, stream=None):
    """forward() that also returns the context for backward(..., saved=):
    (out, state_out, saved), `saved` a uint8 device tensor (allocated if not
    given)."""
    B, N, H, d = q.shape
    frames = gate_logits.shape[1]
    T = 0 if frames == 0 else N // frames
    if frames and N % frames:
        raise ValueError("token axis %d is not a multiple of frames %d" % (N, frames))
    if out is None:
        out = torch.empty_like(q)
    if state_out is None:
        state_out = torch.empty(B, H, d, d + 1, device=q.device, dtype=torch.float32)
    if saved is None:
        n = gla_saved_bytes(B, H, frames, T, d)
        saved = torch.empty(max(n, 1), device=q.device, dtype=torch.uint8)
    gla_forward_train(q, k, v, gate_logits, state_in, state_out, out, saved, B, H, frames, T, d,
                      eps, stream)
    return out, state_out, saved


def backward(q, k, v, gate_logits, dout, state_in=None, dstate_out=None, eps: float = 1e-6,
             stream=None, want_dstate_in: bool = True, saved=None):
    """Convenience wrapper of gla_backward (gla_backward_saved when `saved`,
    the context of forward_train for the same inputs, is given): allocates the
    gradients and returns (dq, dk, dv, dgate_logits, dstate_in or None)."""
    B, N, H, d = q.shape
    frames = gate_logits.shape[1]
    if frames == 0:
        T = 0
    else:
        if N % frames:
            raise ValueError("token axis %d is not a multiple of frames %d" % (N, frames))
        T = N // frames
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dg = torch.empty_like(gate_logits)
    ds_in = (torch.empty(B, H, d, d + 1, device=q.device, dtype=torch.float32)
             if want_dstate_in else None)
    if saved is None:
        gla_backward(q, k, v, gate_logits, state_in, dout, dstate_out, dq, dk, dv, dg, ds_in, B,
                     H, frames, T, d, eps, stream)
    else:
        gla_backward_saved(q, k, v, gate_logits, state_in, saved, dout, dstate_out, dq, dk, dv,
                           dg, ds_in, B, H, frames, T, d, eps, stream)
    return dq, dk, dv, dg, ds_in
