"""B200-native (sm_100a) Jensen-bias-corrected attention over a low-bit (INT2/INT4) KV cache.

Modules: `api` (ctypes binding of libqkv, the C ABI in include/qkv.h), `build` (nvcc build of
libqkv.so in-tree), `workloads` (seeded synthetic inputs). Importing the package loads nothing;
`api.load_library()` loads the CUDA library on first use.
"""
__all__ = ["api", "build", "workloads"]
