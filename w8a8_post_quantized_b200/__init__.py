"""B200-native (sm_100a) ZeroQuant-style W8A8 linear.

The kernels live in the C-ABI library ``libzq.so`` (sources in ``csrc/``,
declarations in ``include/zq.h``); ``w8a8_post_quantized_b200.zq`` is the
thin Python binding with the same function names, and
``w8a8_post_quantized_b200.inputs`` the seeded synthetic workloads.  Importing
the package itself loads nothing, so the workload generators work without a
GPU; importing ``zq`` loads the library and fails loudly if it is missing.
"""
__all__ = ["zq", "inputs", "build"]
