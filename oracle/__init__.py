"""Plain fp64 CPU oracle for latent / grouped KV-cache decode attention.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
CPU-baseline leg of the benchmark -- never by the library itself.  It shares no
code with the CUDA path; its functions are written from the definitions on the
pages (see attend.py for the citations) and pinned by brute force, closed forms
and identities in tests/test_oracle_*.py.
"""
from .attend import (grouped_decode, mla_absorbed_decode, gqla_group_decode, gla_group_decode,
                     gta_group_decode, merge_partials, append_rows, append_destinations, visible_keys,
                     absorb_query, unabsorb_output, expand_latent, output_projection)
from . import accounting
from . import fp8

__all__ = ["grouped_decode", "mla_absorbed_decode", "gqla_group_decode", "gla_group_decode",
           "gta_group_decode", "merge_partials", "append_rows", "append_destinations", "visible_keys",
           "absorb_query", "unabsorb_output", "expand_latent", "output_projection", "accounting", "fp8"]
