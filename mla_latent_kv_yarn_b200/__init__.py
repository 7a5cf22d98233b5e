"""MLA latent-KV decode with YaRN RoPE for NVIDIA B200 (sm_100a).

The compute path is libxmla.so (C ABI in include/xmla.h, CUDA kernels in
csrc/); ``xmla`` is its ctypes binding and ``session`` sequences the calls.
Nothing is imported eagerly so that building does not need a GPU.
"""

__all__ = ["xmla", "session", "workloads", "build"]
