"""B200-native (sm_100a) DeepSeek-V4 CSA/HCA hybrid-attention hot path.

The compute lives in libcsa.so (CUDA kernels behind a C ABI, declared in
include/csa.h); `compressed_sparse_kv_04_b200.binding` is a thin ctypes layer
with the same entry-point names.  The binding loads the library on first use
and raises if it is missing: there is no CPU fallback.
"""
__all__ = ["binding", "configs", "synth"]
