"""FlashPrefill V2 block-sparse prefill attention for NVIDIA B200 (sm_100a).

The product is the C-ABI library ``libfp2.so`` built from ``csrc/`` (its
header is ``include/fp2.h`` at the repository root).  ``binding`` is a thin
ctypes layer over it that marshals torch tensors into pointers; every step
of the path runs in the library's CUDA kernels.  ``synth`` generates seeded
synthetic inputs.  The library is loaded on first use and its absence is an
error: there is no fallback path.
"""

__version__ = "0.1.0"
