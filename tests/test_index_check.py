"""Index validation on the GPU (mla_check_topk_indices, mla_set_index_checks).

The pages' index mask scatters 0 into a -inf row (page "Query-key
similarity", decode excerpt), so a position listed twice is selected once; the
kernels require distinct valid entries and this check reports rows that break
that.  Expected flags come from plain set arithmetic on the host; entries
outside [0, min(end_pos, S_max)) are padding and never count as repeats.
"""
import numpy as np
import pytest
import torch

import sparse_latent_attention_absorb_b200 as pkg
from sparse_latent_attention_absorb_b200 import workloads as wl

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
BAD_INDEX = 5


def expected_flags(end_pos, topk_idx, S_max):
    ep = np.minimum(np.maximum(end_pos.numpy().astype(np.int64), 0), S_max)
    flags = []
    for b, row in enumerate(topk_idx.numpy().astype(np.int64)):
        valid = row[(row >= 0) & (row < ep[b])]
        flags.append(int(len(set(valid.tolist())) != len(valid)))
    return np.array(flags, dtype=np.int32)


def run_check(end_pos, topk_idx, S_max):
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    flags = pkg.mla_check_topk_indices(end_pos.to(DEV), topk_idx.to(DEV), S_max, d_status=status,
                                       row_flags=torch.full((topk_idx.shape[0],), -1, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    return int(status.item()), flags.cpu().numpy()


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_latent_attention_absorb_b200 import build
    build.build()
    pkg.load_library()


@pytest.mark.parametrize("name", list(wl.SMALL_WORKLOADS) + list(wl.WORKLOADS))
def test_generated_index_rows_are_distinct(name):
    w = wl.ALL_WORKLOADS[name]
    gen = torch.Generator().manual_seed(w.seed)
    end_pos, topk_idx = wl.make_indices(w, gen)
    status, flags = run_check(end_pos, topk_idx, w.S_max)
    assert status == 0
    assert flags.tolist() == [0] * w.B


def test_repeats_are_flagged_per_row_and_padding_is_not():
    w = wl.ALL_WORKLOADS["small_b5_ctx40-700_top333"]
    end_pos, topk_idx = wl.make_indices(w, torch.Generator().manual_seed(w.seed))
    idx = topk_idx.clone()
    ep = end_pos.tolist()
    # row 1: a valid entry copied over another valid entry
    idx[1, 3] = idx[1, 0]
    # row 3: a valid entry copied into a padding slot (end_pos < K there)
    r3_pad = int((idx[3] < 0).nonzero()[0]) if (idx[3] < 0).any() else None
    if r3_pad is not None:
        idx[3, r3_pad] = idx[3, 0]
    # row 2: repeated padding values (-1, end_pos, a huge value) stay padding
    idx[2, -3:] = torch.tensor([-1, ep[2], 1 << 30], dtype=torch.int32)
    idx[2, -6:-3] = torch.tensor([-1, ep[2], 1 << 30], dtype=torch.int32)
    status, flags = run_check(end_pos, idx, w.S_max)
    want = expected_flags(end_pos, idx, w.S_max)
    assert flags.tolist() == want.tolist()
    assert want[1] == 1 and want[2] == 0 and want[0] == 0
    assert status == BAD_INDEX


def test_end_pos_beyond_s_max_is_clamped():
    # entries in [S_max, end_pos) are padding: a repeat there is not a repeat
    S = 100
    end_pos = torch.tensor([250, 60], dtype=torch.int32)
    idx = torch.tensor([[5, 120, 120, 7, 99], [59, 60, 60, 61, 0]], dtype=torch.int32)
    status, flags = run_check(end_pos, idx, S)
    assert flags.tolist() == expected_flags(end_pos, idx, S).tolist() == [0, 0]
    assert status == 0
    idx[0, 4] = 7
    status, flags = run_check(end_pos, idx, S)
    assert flags.tolist() == [1, 0] and status == BAD_INDEX


def test_rows_longer_than_one_bitmap_pass():
    # 1,048,576 positions per pass: repeats beyond the first pass, and a pair
    # of entries one pass apart (same bit, different passes: distinct)
    S = 3 * (1 << 20) + 17
    end_pos = torch.tensor([S, S, S], dtype=torch.int32)
    P = 1 << 20
    idx = torch.tensor([[0, P, 2 * P, 3 * P + 16, 5, P + 5],
                        [2 * P + 9, 7, 2 * P + 9, -1, -1, -1],
                        [3 * P + 16, 1, 2, 3, 4, 3 * P + 16]], dtype=torch.int32)
    status, flags = run_check(end_pos, idx, S)
    assert flags.tolist() == expected_flags(end_pos, idx, S).tolist() == [0, 1, 1]
    assert status == BAD_INDEX


def test_status_word_keeps_an_earlier_error():
    w = wl.ALL_WORKLOADS["small_b2_ctx300_top100"]
    end_pos, topk_idx = wl.make_indices(w, torch.Generator().manual_seed(w.seed))
    idx = topk_idx.clone()
    idx[0, 1] = idx[0, 0]
    status = torch.full((1,), 4, dtype=torch.int32, device=DEV)
    pkg.mla_check_topk_indices(end_pos.to(DEV), idx.to(DEV), w.S_max, d_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 4


def test_opt_in_checks_run_before_every_decode():
    d = wl.generate("small_b3_ctx1001_top256")
    g = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    dup = g["topk_idx"].clone()
    dup[2, 10] = dup[2, 11]
    prev = pkg.set_index_checks(True)
    try:
        for idx, want in ((g["topk_idx"], 0), (dup, BAD_INDEX)):
            status = torch.zeros(1, dtype=torch.int32, device=DEV)
            out = pkg.mla_sparse_decode(g["q_nope"], g["q_pe"], g["kv_cache"], g["pe_cache"], g["end_pos"], idx,
                                        g["wkv_b"], g["scale"], d_status=status)
            torch.cuda.synchronize()
            assert int(status.item()) == want
            assert torch.isfinite(out.float()).all()
        pkg.set_index_checks(False)
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        pkg.mla_sparse_decode(g["q_nope"], g["q_pe"], g["kv_cache"], g["pe_cache"], g["end_pos"], dup, g["wkv_b"],
                              g["scale"], d_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0  # off: nothing checks, the decode runs as before
    finally:
        pkg.set_index_checks(prev)
