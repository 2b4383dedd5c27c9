"""Quantized latent-MoE expert layer for B200 (sm_100a).

The layer runs in hand-written CUDA kernels behind the C ABI declared in
``include/elq.h`` (``libelq.so``).  ``quantized_latent_moe_b200.elq`` is the
thin ctypes binding: it marshals torch tensors' device pointers and the current
CUDA stream into those calls and does nothing else.  ``synth`` holds the seeded
synthetic input recipe.
"""
__all__ = ["elq", "synth"]
