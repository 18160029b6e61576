"""Jet-Long dynamic bifocal RoPE attention on B200 (sm_100a).

The compute lives in ``libjetlong.so`` (CUDA kernels behind a C ABI declared in
``include/jetlong.h``).  ``rope_context_extension_sm_b200.jetlong`` is the thin
ctypes binding; it loads the library on import and raises if it is missing.
``rope_context_extension_sm_b200.inputs`` holds the seeded synthetic workloads.
Importing this package itself loads nothing.
"""
__all__ = ["jetlong", "inputs"]
