"""Fused scaled-dot-product attention (forward + deterministic backward) for
NVIDIA B200 (sm_100a): hand-written tcgen05 / TMA kernels behind a C ABI
(include/sdpa.h), with this package as its thin Python binding.

The shared library is loaded on first use; importing the package does not
touch the GPU.
"""
from .binding import (  # noqa: F401
    BWD_ALL,
    BWD_DKDV,
    BWD_DQ,
    BWD_PREPROCESS,
    EXPORTED,
    SdpaError,
    load_library,
    sdpa_bwd,
    sdpa_bwd_bias_grad,
    sdpa_bwd_bias_grad_workspace_size,
    sdpa_bwd_noalloc,
    sdpa_bwd_varlen,
    sdpa_bwd_workspace_size,
    sdpa_debug_wait_timeout,
    sdpa_exp2_fma,
    sdpa_fire_backward,
    sdpa_fire_table,
    sdpa_fwd,
    sdpa_fwd_varlen,
    sdpa_read_device_status,
    sdpa_set_wait_limit_ns,
    sdpa_status_string,
    sdpa_t5_bucket,
)
