"""B200-native JoLT KV-cache compression (partial Tucker + rotated low-bit
residual + joint Lagrangian rank/bit allocation).

`jolt` is the ctypes binding of the CUDA library libjolt.so (C ABI in
include/jolt.h); `synth` makes seeded synthetic caches. The library is loaded
on first use, so importing the package needs no GPU.
"""
from . import jolt, synth  # noqa: F401
