"""Liger Attention forward pass (gated recurrent branch + 64-token sliding-window
softmax attention) for NVIDIA B200 (sm_100a).

The compute lives in the CUDA library ``csrc/`` builds into ``libliger_attn.so``;
``ops`` is a thin ctypes binding over its C ABI (``include/liger_attn.h``).
Importing the package does not load the library: the first call does, and it
raises if the library is missing.  There is no CPU fallback.
"""
__all__ = ["ops", "inputs", "build"]
