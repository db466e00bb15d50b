"""nvfp4_block_numerics_b200 -- a B200-native NVFP4 block-numerics engine.

The compute path lives in ``libnv4.so`` (hand-written sm_100a CUDA kernels behind
a C ABI, declared in ``include/nv4.h``).  ``binding`` marshals torch tensors into
that ABI; ``inputs`` generates the seeded synthetic workloads.  The CUDA library
is loaded lazily, on first use of the binding, and a missing library is an error.
"""
