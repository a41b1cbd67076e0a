"""B200-native decode megakernel for parallel-layer MoE decoders.

The decode step runs in ``libmk.so`` (CUDA, sm_100a) behind the C ABI in
``include/mk.h``; ``engine.Decoder`` is the Python handle on it.
"""

__all__ = ["configs", "synth", "engine", "mk", "roofline"]
