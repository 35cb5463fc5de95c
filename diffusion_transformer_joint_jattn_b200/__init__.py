"""B200-native joint attention for diffusion transformers.

``jattn``      ctypes binding of libjattn.so (the CUDA path; no CPU fallback)
``workloads``  seeded synthetic inputs shared by the tests and the benchmark
``build``      nvcc build step for libjattn.so (sm_100a)
"""
__all__ = ["jattn", "workloads", "build"]
