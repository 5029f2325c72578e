"""B200-native (sm_100a) Q8_0 single-token decode and fused MoE up/gate + SwiGLU.

The kernels and their C ABI live in ``csrc/`` (built into ``libq8.so``; the
header is ``include/q8.h``); ``q8`` is the thin ctypes binding; ``synth``
draws the seeded synthetic inputs.  Importing the package loads nothing;
``moe_up_gate_b200.q8.load()`` loads (and if needed builds) the library.
"""
__all__ = ["q8", "synth", "build"]
