"""B200-native sliced r-bit (Matryoshka) linear layers.

The CUDA library and its ctypes binding live in ``matq``; ``synth`` draws seeded inputs.
"""
