"""fp64 CPU oracle of the absorbed, top-k masked MLA decode step and of the
attention output projection that follows it.

TEST INFRASTRUCTURE ONLY: imported by the tests, ``__graft_entry__.smoke()``
and the benchmark's CPU-baseline leg, never by the CUDA package.
"""
from .oracle import OracleResult, build, mla_sparse_decode, num_threads, output_projection

__all__ = ["OracleResult", "build", "mla_sparse_decode", "num_threads", "output_projection"]
