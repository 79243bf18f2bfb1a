"""B200-native Streaming Sortformer diarization engine.

The engine is libsf.so (C ABI in include/sf.h, CUDA kernels for sm_100a in
csrc/); ``binding`` exposes its calls under the same names.
"""
__all__ = ["binding", "build"]
