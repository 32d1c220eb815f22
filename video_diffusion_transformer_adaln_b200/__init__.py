"""B200-native forward pass of a gated-AdaLN DiT block over video latent tokens.

The compute lives in the CUDA library ``_lib/libh3b.so`` (C ABI in
``include/h3b.h``); ``h3b`` is its ctypes binding, ``synth`` the seeded
synthetic workloads, ``runtime`` the device-side helpers that hold a block's
weights and workspace.
"""
__all__ = ["h3b", "synth", "runtime"]
