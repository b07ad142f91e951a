"""B200-native differentiable tile rasterizer for 3D Gaussian Splatting.

The compute path is the C-ABI CUDA library ``libgs.so`` (sources in ``csrc/``,
declarations in ``include/gs.h``); ``abi`` is its thin ctypes binding and
``pipeline`` marshals torch device buffers through it.  ``scenes`` draws the
seeded synthetic inputs.  Importing the package loads nothing; the library is
loaded on first use and a missing build is an error, never a fallback.
"""
__all__ = ["abi", "pipeline", "scenes"]
