"""B200-native (sm_100a) QUADS rollout hot path: NVFP4 online activation
quantization with residual channel scoring and top-k selection, the grouped
W4A4 MoE expert GEMM with Residual Activation Compensation on tcgen05, and
the trainer-side NVFP4 weight quantize-dequantize.

The compute lives in ``libnvfp4_quads.so`` (C ABI: include/nvfp4_quads.h);
``api`` marshals torch tensors into it and ``moe`` strings the calls into a
layer.  Importing this package does not load the library; the first call does,
and raises if it is not built.
"""
from . import workloads  # noqa: F401  (pure-Python input generators)

__all__ = ["api", "moe", "workloads", "build"]


def build():
    from .build import build as _b
    return _b()
