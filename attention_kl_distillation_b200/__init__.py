"""B200-native fused attention-KL divergence (StreamKL forward and recompute backward).

The compute path is libstreamkl.so (sm_100a kernels behind a C ABI, see
include/streamkl.h); ``streamkl`` is its thin Python binding.
"""
from .binding import (StreamKLError, bwd, bwd_algorithm_for, bwd_noalloc, fwd,  # noqa: F401
                      fwd_splitk, launch_count, query_device_status, set_bwd_algorithm,
                      set_wait_limit_ms, splitk_suggest, splitk_workspace_size, streamkl,
                      workspace_size)
