"""NVFP4 weight-streaming decode round for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libnvfp4decode.so`` (CUDA kernels,
see ``include/nvfp4decode.h``).  ``abi`` is its thin ctypes binding; it loads
the library on first use and raises if it is missing -- there is no fallback.
``synth`` holds the seeded synthetic input generators.
"""

__all__ = ["abi", "synth"]
