"""kv2d: dynamic two-dimensional KV-cache compression and decode attention
over the compressed cache, as CUDA kernels for NVIDIA B200 (sm_100a) behind a
C ABI (include/kv2d.h).  This package holds the ctypes binding (binding.py),
the in-tree build step (build.py), the CUDA sources (csrc/) and the seeded
synthetic input generator (synth.py)."""
