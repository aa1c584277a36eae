"""B200-native AdamW step with FP8-stored moments (m in E4M3, v in E5M2).

The optimizer runs in ``libfp8adam.so`` (CUDA, sm_100a) behind the C ABI of
include/fp8adam.h; ``capi`` binds it with ctypes and ``FP8AdamW`` wraps it
for torch tensors.  ``workloads`` draws seeded synthetic inputs.
"""
from . import capi  # noqa: F401
from .optim import FP8AdamW  # noqa: F401

__all__ = ["capi", "FP8AdamW"]
