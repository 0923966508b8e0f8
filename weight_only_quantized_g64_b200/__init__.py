"""weight_only_quantized_g64_b200 -- B200-native weight-only group-64 quantized projections.

The compute lives in librq.so (hand-written sm_100a CUDA kernels behind the C
ABI declared in include/rq.h); ``rq`` holds the thin ctypes binding.
"""
