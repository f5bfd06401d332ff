"""Routed sparse-MoE block (router, top-k, low-bit SwiGLU experts, shared
expert, weighted combine) on B200 (sm_100a).

Importing the package loads nothing compiled.  The CUDA path lives behind the
C ABI in ``include/moe.h`` and is reached through :mod:`.moe` (ctypes binding);
the seeded synthetic inputs come from :mod:`.synth`.
"""

__all__ = ["moe", "synth"]
