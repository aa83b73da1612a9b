"""Failure detection: every device wait is bounded.  The self-test kernel
waits, through the kernels' own wait(), on a barrier that nothing arrives on:
it must give up after the limit (2 s), report MLA_ERR_DEVICE_TIMEOUT in the
status word and leave the context usable.  No fault, trap or hang is caused:
the wait runs out and the kernel returns."""
import ctypes
import time

import numpy as np
import pytest
import torch

import sparse_latent_attention_absorb_b200 as pkg
from sparse_latent_attention_absorb_b200 import binding, build

TIMEOUT = 4  # MLA_ERR_DEVICE_TIMEOUT


def test_selftest_rejects_bad_arguments_without_a_launch():
    build.build()
    lib = binding.load_library()
    A = 0x10000
    assert lib.mla_selftest_wait_timeout(None, ctypes.c_void_p(A), None) == 1
    assert lib.mla_selftest_wait_timeout(ctypes.c_void_p(A), None, None) == 1
    assert lib.mla_selftest_wait_timeout(ctypes.c_void_p(A + 2), ctypes.c_void_p(A), None) == 1


@pytest.mark.gpu
def test_bounded_wait_gives_up_reports_and_leaves_the_context_usable():
    import oracle
    from sparse_latent_attention_absorb_b200 import workloads as wl
    t0 = time.perf_counter()
    status, result = binding.selftest_wait_timeout()
    elapsed = time.perf_counter() - t0
    assert status == TIMEOUT
    assert result == 4  # gave up, set the abort flag, the second wait returned at once
    assert 1.5 < elapsed < 60
    # the context still runs the decode correctly
    d = wl.generate("small_b3_ctx1001_top256")
    dev = torch.device("cuda:0")
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    out = pkg.mla_sparse_decode(g["q_nope"], g["q_pe"], g["kv_cache"], g["pe_cache"], g["end_pos"], g["topk_idx"],
                                g["wkv_b"], g["scale"])
    torch.cuda.synchronize()
    ref = oracle.mla_sparse_decode(d["q_nope"], d["q_pe"], d["kv_cache"], d["pe_cache"], d["end_pos"],
                                   d["topk_idx"], d["wkv_b"], d["scale"]).out
    assert np.max(np.abs(out.double().cpu().numpy() - ref)) <= 1e-2 * np.max(np.abs(ref)) + 1e-3
