"""B200-native MoE expert-parallel dispatch / combine.

The hot path (routing layout, FP8/BF16 dispatch, combine and both backward
passes) runs in the CUDA library ``libep_b200.so`` behind the C ABI declared
in ``include/ep.h``; ``combine_ep_get_histogram_b200.ep`` is its thin ctypes
binding.  ``workloads`` draws the seeded synthetic inputs.
"""
