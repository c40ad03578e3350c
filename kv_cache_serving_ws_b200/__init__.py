"""B200-native unit step of the Wan-Streamer v0.2 performer.

The hot path (K/V cache append, block-causal unit attention, Euler update) runs
in the CUDA library libws.so behind the C ABI of include/ws.h; ``native`` is its
thin ctypes binding, ``synth`` the seeded synthetic-input generator.
"""
from . import native  # noqa: F401
