"""fp64 CPU oracle of the absorbed, top-k masked MLA decode step.

TEST INFRASTRUCTURE ONLY: imported by the tests, ``__graft_entry__.smoke()``
and the benchmark's CPU-baseline leg, never by the CUDA package.
"""
from .oracle import OracleResult, build, mla_sparse_decode, num_threads

__all__ = ["OracleResult", "build", "mla_sparse_decode", "num_threads"]
