"""B200-native kernelized linear attention.

The compute lives in liblinattn.so (hand-written CUDA for sm_100a behind the
C ABI in include/la_api.h); ``api`` is its thin Python binding and
``inputs`` draws the seeded synthetic tensors used by tests and benchmarks.
"""
from .api import (  # noqa: F401
    LinearAttention,
    LinearAttentionError,
    la_backward,
    la_decode_step,
    la_forward,
    la_get_device_error,
    la_launch_count,
    la_profile_collect,
    la_profile_enable,
    la_status_string,
    la_version,
    la_workspace_size,
    load_library,
)
