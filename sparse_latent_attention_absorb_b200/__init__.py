"""Sparse absorbed MLA decode for B200 (sm_100a).

DeepSeek-V3.2-Exp's multi-head latent attention decode step with the
indexer's top-k mask (and the output projection wo that follows it),
computed by hand-written tcgen05/TMEM kernels behind a
small C ABI (include/mla_sparse_decode.h).  ``binding`` holds the Python entry
points (argument marshalling only); ``workloads`` the seeded synthetic inputs.
The CUDA library is loaded on first use and its absence is an error.
"""
from .binding import (Fp8Wkvb, MLAError, PreparedWo, host_workspace_size, load_library, mla_absorb_q,
                      mla_check_topk_indices, mla_combine_value_up, mla_dequant_fp8_blocks,
                      mla_output_projection, mla_output_projection_prepared, mla_output_projection_shard,
                      mla_prepare_wo, mla_sparse_attend, mla_sparse_decode, mla_sparse_decode_heads,
                      mla_sparse_decode_host, mla_sparse_decode_project, mla_sparse_prefill, num_splits,
                      project_workspace_size, projection_workspace_size, set_index_checks, workspace_size)

__all__ = ["Fp8Wkvb", "MLAError", "PreparedWo", "host_workspace_size", "load_library", "mla_absorb_q",
           "mla_check_topk_indices", "mla_combine_value_up", "mla_dequant_fp8_blocks",
           "mla_output_projection", "mla_output_projection_prepared", "mla_output_projection_shard",
           "mla_prepare_wo", "mla_sparse_attend", "mla_sparse_decode", "mla_sparse_decode_heads",
           "mla_sparse_decode_host", "mla_sparse_decode_project", "mla_sparse_prefill", "num_splits",
           "project_workspace_size", "projection_workspace_size", "set_index_checks", "workspace_size"]
