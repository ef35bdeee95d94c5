"""persistent_task_runtime_b200: one whole transformer decode step as a single
persistent sm_100a megakernel, behind a small C ABI (``include/mk.h``).

The native library is loaded on first use by :mod:`.mk` (ctypes binding).
There is no CPU fallback: if the library is missing or no GPU is present the
calls raise.
"""

__all__ = ["mk", "synth", "kvcache"]
