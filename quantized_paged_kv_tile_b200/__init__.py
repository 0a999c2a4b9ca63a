"""B200 (sm_100a) variance-normalized, tile-quantized paged KV cache.

Modules: ``kvq`` (ctypes binding over the C ABI in include/kvq.h),
``paged`` (host-side bookkeeping of a paged cache), ``synth`` (seeded
synthetic workloads), ``build`` (nvcc build of libkvq.so).
"""
