"""Tensor-parallel decode (page "Queries", MLA constructor: wkv_b is a
ColumnParallelLinear, so a rank holds 128 / world_size heads; wo is a
RowParallelLinear whose partial outputs the ranks sum).

CPU (not gpu): the head split and the slicing of queries, wkv_b and wo, and
the whole shard -> partial projection -> all-reduce chain over two gloo ranks,
each rank's arithmetic done by the fp64 oracle, against the oracle's decode
and projection of all 128 heads.

GPU: every shard of 2, 4 and 8 ranks through the C ABI
(mla_sparse_decode_heads, mla_output_projection_shard) against the oracle
restricted to the shard's heads, and the ranks' partial projections summed.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from sparse_latent_attention_absorb_b200 import tp
from sparse_latent_attention_absorb_b200 import workloads as wl

DIM = 256  # projection width of the CPU cases (the pages' 7168 on the GPU)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_head_ranges_cover_the_heads_once():
    for world in (1, 2, 4, 8, 16, 32, 64, 128):
        seen = []
        for r in range(world):
            h0, h1 = tp.head_range(world, r)
            assert h1 - h0 == 128 // world
            seen.extend(range(h0, h1))
        assert seen == list(range(128))
    with pytest.raises(ValueError):
        tp.head_range(3, 0)
    with pytest.raises(ValueError):
        tp.head_range(2, 2)


def test_shard_slices_queries_wkv_b_and_wo():
    d = wl.generate("small_b2_ctx300_top100", caches=False)
    wo = wl.generate_projection(1, DIM, seed=7)["wo"]
    for world, rank in ((2, 1), (4, 2), (8, 7)):
        s = tp.shard(world, rank, d["q_nope"], d["q_pe"], d["wkv_b"], wo)
        h0, h1 = s["heads"]
        assert torch.equal(s["q_nope"], d["q_nope"][:, h0:h1]) and s["q_nope"].is_contiguous()
        assert torch.equal(s["q_pe"], d["q_pe"][:, h0:h1]) and s["q_pe"].is_contiguous()
        # wkv_b rows of head h are [256 h, 256 h + 256): W_UK then W_UV
        assert torch.equal(s["wkv_b"], d["wkv_b"][256 * h0:256 * h1]) and s["wkv_b"].is_contiguous()
        # wo columns of head h are [128 h, 128 h + 128) (x.flatten(2): k = 128 h + e)
        assert torch.equal(s["wo"], wo[:, 128 * h0:128 * h1])
        assert s["wo"].stride() == (16384, 1)


def _oracle_decode(q_nope, q_pe, kv, pe, end_pos, topk, wkv_b, scale):
    return torch.from_numpy(oracle.mla_sparse_decode(q_nope, q_pe, kv, pe, end_pos, topk, wkv_b, scale).out)


def _oracle_project(x, wo):
    # x: the oracle decode's float64 output; wo: a bf16 column slice
    return torch.from_numpy(oracle.output_projection(x.to(torch.float64), wo.to(torch.float64)))


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), OMP_NUM_THREADS="2")
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        d = wl.generate("small_b2_ctx300_top100")
        wo = wl.generate_projection(1, DIM, seed=7)["wo"]
        sh = tp.shard(world, rank, d["q_nope"], d["q_pe"], d["wkv_b"], wo)
        delta, out_r = tp.decode_project(sh, d["kv_cache"], d["pe_cache"], d["end_pos"], d["topk_idx"], d["scale"],
                                         decode=_oracle_decode, project=_oracle_project)
        torch.save({"delta": delta, "out_r": out_r, "heads": sh["heads"]}, os.path.join(out_dir, f"rank{rank}.pt"))
        torch.distributed.barrier()
    finally:
        torch.distributed.destroy_process_group()


def test_shard_partial_projection_all_reduce_over_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn",
                       join=True)
    d = wl.generate("small_b2_ctx300_top100")
    wo = wl.generate_projection(1, DIM, seed=7)["wo"]
    full = oracle.mla_sparse_decode(d["q_nope"], d["q_pe"], d["kv_cache"], d["pe_cache"], d["end_pos"],
                                    d["topk_idx"], d["wkv_b"], d["scale"])
    want = oracle.output_projection(torch.from_numpy(full.out), wo.to(torch.float64))
    for r in range(world):
        got = torch.load(tmp_path / f"rank{r}.pt")
        h0, h1 = got["heads"]
        # each rank's heads are those heads of the full decode
        np.testing.assert_allclose(got["out_r"].numpy(), full.out[:, h0:h1], rtol=1e-12, atol=1e-14)
        # after the all-reduce every rank holds the projection of all heads
        np.testing.assert_allclose(got["delta"].numpy(), want, rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- GPU

DEV = torch.device("cuda:0")


@pytest.mark.gpu
@pytest.mark.parametrize("world", [2, 4, 8])
@pytest.mark.parametrize("name", ["small_b4_ctx600-2k_recent128_top400", "small_b80_ctx700_top300"])
def test_decode_shards_match_the_oracle_on_their_heads(world, name):
    d = wl.generate(name)
    g = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    ref = oracle.mla_sparse_decode(d["q_nope"], d["q_pe"], d["kv_cache"], d["pe_cache"], d["end_pos"],
                                   d["topk_idx"], d["wkv_b"], d["scale"])
    for rank in range(world):
        s = tp.shard(world, rank, g["q_nope"], g["q_pe"], g["wkv_b"])
        h0, h1 = s["heads"]
        lse = torch.full((d["q_nope"].shape[0], h1 - h0), float("nan"), dtype=torch.float32, device=DEV)
        from sparse_latent_attention_absorb_b200 import binding
        out = binding.mla_sparse_decode_heads(s["q_nope"], s["q_pe"], g["kv_cache"], g["pe_cache"], g["end_pos"],
                                              g["topk_idx"], s["wkv_b"], g["scale"], lse_out=lse)
        torch.cuda.synchronize()
        want = ref.out[:, h0:h1]
        got = out.double().cpu().numpy()
        assert np.all(np.isfinite(got))
        assert np.max(np.abs(got - want)) <= 1e-2 * np.max(np.abs(want)) + 1e-3
        assert np.max(np.abs(lse.double().cpu().numpy() - ref.lse[:, h0:h1])) <= 1e-2


@pytest.mark.gpu
def test_all_heads_through_the_shard_entry_equal_the_decode():
    import sparse_latent_attention_absorb_b200 as pkg
    from sparse_latent_attention_absorb_b200 import binding
    d = wl.generate("small_b5_ctx40-700_top333")
    g = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    a = pkg.mla_sparse_decode(g["q_nope"], g["q_pe"], g["kv_cache"], g["pe_cache"], g["end_pos"], g["topk_idx"],
                              g["wkv_b"], g["scale"])
    b = binding.mla_sparse_decode_heads(g["q_nope"], g["q_pe"], g["kv_cache"], g["pe_cache"], g["end_pos"],
                                        g["topk_idx"], g["wkv_b"], g["scale"])
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.gpu
@pytest.mark.parametrize("n_heads", [1, 3, 40, 127])
def test_uneven_head_counts(n_heads):
    from sparse_latent_attention_absorb_b200 import binding
    d = wl.generate("small_b3_ctx1001_top256")
    h0 = 128 - n_heads
    qn, qp = d["q_nope"][:, h0:].contiguous(), d["q_pe"][:, h0:].contiguous()
    wb = d["wkv_b"][256 * h0:].contiguous()
    ref = oracle.mla_sparse_decode(qn, qp, d["kv_cache"], d["pe_cache"], d["end_pos"], d["topk_idx"], wb, d["scale"])
    out = binding.mla_sparse_decode_heads(qn.to(DEV), qp.to(DEV), d["kv_cache"].to(DEV), d["pe_cache"].to(DEV),
                                          d["end_pos"].to(DEV), d["topk_idx"].to(DEV), wb.to(DEV), d["scale"])
    torch.cuda.synchronize()
    got = out.double().cpu().numpy()
    assert got.shape == ref.out.shape
    assert np.max(np.abs(got - ref.out)) <= 1e-2 * np.max(np.abs(ref.out)) + 1e-3


@pytest.mark.gpu
@pytest.mark.parametrize("world", [2, 4, 8])
@pytest.mark.parametrize("B", [3, 64])
def test_row_parallel_partials_sum_to_the_projection(world, B):
    from sparse_latent_attention_absorb_b200 import binding
    dim = wl.D_MODEL
    p = wl.generate_projection(B, dim, seed=4100 + B)
    x, wo = p["x"], p["wo"]
    xg, wog = x.to(DEV), wo.to(DEV)
    total = np.zeros((B, dim))
    bound = np.zeros((B, dim))
    for rank in range(world):
        h0, h1 = tp.head_range(world, rank)
        xs = xg.view(B, 128, 128)[:, h0:h1].reshape(B, -1).contiguous()
        ws = wog[:, 128 * h0:128 * h1]  # a strided column slice of the full wo
        delta = binding.mla_output_projection_shard(xs, ws)
        torch.cuda.synchronize()
        want = oracle.output_projection(x.view(B, 128, 128)[:, h0:h1].reshape(B, -1).contiguous(),
                                        wo[:, 128 * h0:128 * h1].contiguous())
        got = delta.double().cpu().numpy()
        # one bf16 rounding of an fp32 sum over the shard's inputs
        tol = 2.0 ** -8 * np.abs(want) + 1e-4 * np.max(np.abs(want))
        assert np.all(np.abs(got - want) <= tol)
        total += got
        bound += tol
    full = oracle.output_projection(x, wo)
    # the sum of the ranks' bf16 partials (what the all-reduce adds) against
    # the projection of all heads: the ranks' rounding errors add up
    assert np.all(np.abs(total - full) <= bound + 1e-9 * np.max(np.abs(full)))
