"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the bench.

This package draws random numbers and lays out workload *structure* (how many
sequences, their lengths, which sequences share a prefix, the order in which
the block pool hands out physical blocks).  It holds none of the method's
arithmetic: no slot or block-index computation, no attention maths.  Both the
CPU oracle and the CUDA path start from what it returns and derive everything
else on their own.
"""

from .synth import (CONFIGS, RopeCase, Workload, fill_cache_blocks, make_custom, make_prefix_groups, make_rope_case,
                    make_workload, new_token_positions, ops_for, rope_tables)

__all__ = ["CONFIGS", "Workload", "make_workload", "make_custom", "fill_cache_blocks", "ops_for", "RopeCase",
           "make_rope_case", "new_token_positions", "rope_tables", "make_prefix_groups"]
