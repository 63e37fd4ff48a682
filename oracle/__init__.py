"""fp64 CPU oracle of the Gated DeltaNet mixer, the gated full-attention decode
step and the routed-expert MoE block -- test infrastructure only.

Only the tests, the smoke check and the benchmark's CPU-baseline leg use it.
"""
from .oracle import (AttnResult, MoeRoute, Result, build, gate_from_raw, gated_attn_decode,
                     gdr_bruteforce, gdr_chunked, gdr_recurrent, load, moe_forward, moe_route,
                     rmsnorm_gated, rope_partial)

__all__ = ["Result", "AttnResult", "build", "load", "gdr_recurrent", "gdr_chunked",
           "gdr_bruteforce", "rmsnorm_gated", "gate_from_raw", "rope_partial",
           "gated_attn_decode", "MoeRoute", "moe_route", "moe_forward"]
