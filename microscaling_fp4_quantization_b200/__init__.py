"""fp4q: fused block-Hadamard rotation + microscaling FP4 (MXFP4 / NVFP4) quantization
of bf16 activation rows on NVIDIA B200 (sm_100a).

The compute path lives in hand-written CUDA kernels behind a C ABI (``include/fp4q.h``),
built into ``lib/libfp4q.so``.  ``fp4q`` (this package's binding module) loads that
library with ctypes and raises if it is missing: there is no CPU fallback.

``workloads`` holds the seeded synthetic activation generators; it contains none of the
quantizer's arithmetic.

Importing the package itself loads nothing; ``from microscaling_fp4_quantization_b200 import fp4q``
loads the native library.
"""

__all__ = ["fp4q", "workloads"]
