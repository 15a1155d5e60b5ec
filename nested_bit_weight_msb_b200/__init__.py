"""B200-native sliced r-bit (Matryoshka) linear layers.

The CUDA library and its ctypes binding live in ``matq``; ``mixnmatch`` picks a width per layer
for a budget of effective bits (host logic); ``synth`` draws seeded inputs.
"""
