"""B200-native fused attention-KL divergence (StreamKL forward and recompute backward).

The compute path is libstreamkl.so (sm_100a kernels behind a C ABI, see
include/streamkl.h); ``streamkl`` is its thin Python binding.
"""
from .binding import (StreamKLError, bwd, bwd_algorithm_for, fwd, fwd_splitk, launch_count,  # noqa: F401
                      query_device_status, set_bwd_algorithm, set_wait_limit_ms, streamkl,
                      workspace_size)
