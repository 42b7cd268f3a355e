"""B200-native TACT-KV visual-KV transform codec (CUDA kernels for sm_100a behind a C ABI).

`dct_transform_coding_b200.tactkv` is the binding of libtactkv.so (include/tactkv.h);
`dct_transform_coding_b200.workloads` generates the seeded synthetic inputs.  Importing the
package itself loads nothing native, so input generation works on machines without the library.
"""
__all__ = ["tactkv", "workloads"]
