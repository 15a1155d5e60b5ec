"""fp64 CPU oracle for the sliced r-bit linear layer (test infrastructure only).

Imported only by ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline / reference legs.  It shares no code with the CUDA library.
"""
from .matq_oracle import *  # noqa: F401,F403
from .matq_oracle import (C_BITS, WIDTHS, MODES, prefix, delta, reconstruct, dequant,  # noqa: F401
                          linear, linear_loops, linear_group_sums, bits_read_per_weight,
                          rmsnorm, silu, gated_product, ffn_block, mixnmatch_effective_bits,
                          choose_codes)
