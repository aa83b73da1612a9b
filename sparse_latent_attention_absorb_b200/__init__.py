"""Sparse absorbed MLA decode for B200 (sm_100a).

DeepSeek-V3.2-Exp's multi-head latent attention decode step with the
indexer's top-k mask, computed by hand-written tcgen05/TMEM kernels behind a
small C ABI (include/mla_sparse_decode.h).  ``binding`` holds the Python entry
points (argument marshalling only); ``workloads`` the seeded synthetic inputs.
The CUDA library is loaded on first use and its absence is an error.
"""
from .binding import (MLAError, host_workspace_size, load_library, mla_absorb_q, mla_combine_value_up,
                      mla_sparse_attend, mla_sparse_decode, mla_sparse_decode_host, num_splits, workspace_size)

__all__ = ["MLAError", "host_workspace_size", "load_library", "mla_absorb_q", "mla_combine_value_up",
           "mla_sparse_attend", "mla_sparse_decode", "mla_sparse_decode_host", "num_splits", "workspace_size"]
