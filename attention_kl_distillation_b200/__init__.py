"""B200-native fused attention-KL divergence (StreamKL forward and recompute backward).

The compute path is libstreamkl.so (sm_100a kernels behind a C ABI, see
include/streamkl.h); ``streamkl`` is its thin Python binding.

The library is loaded on first use of one of the names below, not on import
of the package: ``attention_kl_distillation_b200.inputs`` and
``attention_kl_distillation_b200.parallel`` carry no CUDA code and can be
imported in a process that must not map the library.
"""
import importlib

_BINDING_NAMES = ("StreamKLError", "bwd", "bwd_algorithm_for", "bwd_noalloc", "fwd", "fwd_splitk",
                  "launch_count", "query_device_status", "set_bwd_algorithm", "set_wait_limit_ms",
                  "splitk_suggest", "splitk_workspace_size", "streamkl", "workspace_size")

__all__ = list(_BINDING_NAMES)


def __getattr__(name):
    if name in _BINDING_NAMES:
        return getattr(importlib.import_module(".binding", __name__), name)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")
