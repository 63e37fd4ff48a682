"""fp64 CPU oracle of the Gated DeltaNet mixer -- test infrastructure only.

Only the tests, the smoke check and the benchmark's CPU-baseline leg use it.
"""
from .oracle import (Result, build, gate_from_raw, gdr_bruteforce, gdr_chunked, gdr_recurrent,
                     load, rmsnorm_gated)

__all__ = ["Result", "build", "load", "gdr_recurrent", "gdr_chunked", "gdr_bruteforce",
           "rmsnorm_gated", "gate_from_raw"]
