"""The allocation-free entry point, mla_sparse_decode_noalloc.

It serves callers that cannot allocate device memory when they call (a plugin
whose host framework owns the device memory, a loop that must not call
cudaMalloc).  Its scratch is a fixed array inside the library, so these tests
check, through the C ABI, that two calls in a row give the output of the
allocating entry point, and that sizes past the array are refused.  This file
is collected last so that a run that stops at the first failure has already
run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import sparse_latent_attention_absorb_b200 as pkg
from sparse_latent_attention_absorb_b200 import binding
from sparse_latent_attention_absorb_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


# the last case is the largest configuration the fixed scratch is sized for
# (B = 64 rows, K = 2048)
@pytest.mark.parametrize("name", ["small_b4_ctx600-2k_recent128_top400", "b8_ctx4096_top2048",
                                  "b64_ctx1k-32k_top2048"])
def test_noalloc_matches_allocating_entry_point_twice(name):
    lib = pkg.load_library()
    d = wl.generate(name)
    g = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    B, K, S = d["q_nope"].shape[0], d["topk_idx"].shape[1], d["kv_cache"].shape[1]
    assert pkg.workspace_size(B, K, S) <= binding.STATIC_SCRATCH_BYTES
    lse_ref = torch.empty((B, 128), dtype=torch.float32, device=DEV)
    ref = pkg.mla_sparse_decode(g["q_nope"], g["q_pe"], g["kv_cache"], g["pe_cache"], g["end_pos"], g["topk_idx"],
                                g["wkv_b"], g["scale"], lse_out=lse_ref)
    torch.cuda.synchronize()
    ref_np = ref.double().cpu().numpy()
    bound = 1e-2 * float(np.max(np.abs(ref_np))) + 1e-3
    stream = torch.cuda.current_stream()
    for _ in range(2):
        out = torch.full((B, 128, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
        lse = torch.full((B, 128), float("nan"), dtype=torch.float32, device=DEV)
        rc = lib.mla_sparse_decode_noalloc(_p(g["q_nope"]), _p(g["q_pe"]), _p(g["kv_cache"]), _p(g["pe_cache"]),
                                           _p(g["end_pos"]), _p(g["topk_idx"]), _p(g["wkv_b"]),
                                           ctypes.c_float(g["scale"]), _p(out), B, K, S, _p(lse), None,
                                           ctypes.c_void_p(stream.cuda_stream))
        assert rc == 0, binding.STATUS.get(rc, rc)
        torch.cuda.synchronize()
        got = out.double().cpu().numpy()
        assert np.all(np.isfinite(got))
        assert np.max(np.abs(got - ref_np)) <= bound
        assert np.max(np.abs(lse.double().cpu().numpy() - lse_ref.double().cpu().numpy())) <= 1e-2


def test_noalloc_refuses_sizes_past_its_scratch():
    lib = pkg.load_library()
    B, K, S = 4096, 2048, 4096  # needs far more than the fixed scratch
    assert pkg.workspace_size(B, K, S) > binding.STATIC_SCRATCH_BYTES
    fake = ctypes.c_void_p(1 << 20)  # aligned, never dereferenced: refused before any launch
    rc = lib.mla_sparse_decode_noalloc(fake, fake, fake, fake, fake, fake, fake, ctypes.c_float(0.07), fake, B, K, S,
                                       None, None, None)
    assert rc == 2  # MLA_ERR_WORKSPACE
