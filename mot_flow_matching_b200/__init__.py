"""B200-native gen-tower attention layer of a Mixture-of-Transformers
pixel-space flow-matching model (forward + LoRA-training backward).

The compute path is libmotattn.so (hand-written sm_100a kernels behind a C
ABI, include/mot_attn.h); this package holds the build script, the ctypes
binding and the seeded synthetic input generator. Importing the package does
not load the library; the first call into ``layer`` does, and fails loudly if
it is missing.
"""

__all__ = ["synth", "layer", "build"]
