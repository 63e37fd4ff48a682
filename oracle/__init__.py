"""fp64 CPU oracle of the Gated DeltaNet mixer and of the gated full-attention
decode step -- test infrastructure only.

Only the tests, the smoke check and the benchmark's CPU-baseline leg use it.
"""
from .oracle import (AttnResult, Result, build, gate_from_raw, gated_attn_decode, gdr_bruteforce,
                     gdr_chunked, gdr_recurrent, load, rmsnorm_gated, rope_partial)

__all__ = ["Result", "AttnResult", "build", "load", "gdr_recurrent", "gdr_chunked",
           "gdr_bruteforce", "rmsnorm_gated", "gate_from_raw", "rope_partial",
           "gated_attn_decode"]
