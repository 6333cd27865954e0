"""B200 (sm_100a) block-causal gated linear attention: a C-ABI CUDA library
(libgla.so) with a thin Python binding.  See include/gla.h for the ABI."""

from ._binding import (  # noqa: F401
    EXPORTED,
    GLA_ERR_ALIGN,
    GLA_ERR_ALLOC,
    GLA_ERR_DEVICE,
    GLA_ERR_LAUNCH,
    GLA_ERR_NULL,
    GLA_ERR_ROPE,
    GLA_ERR_SCRATCH,
    GLA_ERR_SHAPE,
    GLA_ERR_UNSUPPORTED_D,
    GLA_OK,
    GLAError,
    RopeConfig,
    backward,
    forward,
    forward_gdn,
    forward_rope,
    gla_backward,
    gla_backward_timed,
    gla_device_fault,
    gla_error_string,
    gla_forward,
    gla_forward_gdn,
    gla_forward_gdn_timed,
    gla_forward_noalloc,
    gla_forward_rope,
    gla_forward_rope_timed,
    gla_forward_timed,
    gla_softmax_anchor,
    gla_softmax_anchor_timed,
    gla_noalloc_scratch_bytes,
    gla_trim_workspace,
    gla_version,
    load_library,
    rope_config,
    softmax_anchor,
)

# Every entry point loads libgla.so on first use and raises ImportError when
# it is missing; there is no other implementation to fall back on.
