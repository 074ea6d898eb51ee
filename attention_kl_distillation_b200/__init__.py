"""B200-native fused attention-KL divergence (StreamKL forward and recompute backward).

The compute path is libstreamkl.so (sm_100a kernels behind a C ABI, see
include/streamkl.h); ``streamkl`` is its thin Python binding.
"""
from .binding import (StreamKLError, bwd, fwd, launch_count, query_device_status,  # noqa: F401
                      set_wait_limit_ms, streamkl, workspace_size)
