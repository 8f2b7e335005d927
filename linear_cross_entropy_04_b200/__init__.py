"""B200-native fused linear cross-entropy (FLCE).

The compute path is the CUDA library libflce.so (built in-tree by
`python -m linear_cross_entropy_04_b200.build`); this package only marshals
arguments to its C ABI (include/flce.h). Importing the package does not load
the library; the first call does, and raises if it is missing.
"""

__all__ = [
    "fused_linear_cross_entropy", "cross_entropy", "count_valid", "gemm_bf16", "plan", "scale_grad_",
    "device_error", "phase_times", "FusedLinearCrossEntropyLoss",
    "forward_keep", "backward_from_kept", "keep_workspace_bytes", "KeptLogits",
]


def __getattr__(name):
    if name in __all__:
        from . import api

        return getattr(api, name)
    raise AttributeError(name)
