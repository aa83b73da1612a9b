"""The output projection from a prepared wo (mla_prepare_wo +
mla_output_projection_prepared): the same projection as the page "Attention
update" computes (delta = x . wo^T, wo [dim, 16384], the pages' dim 7168),
from a copy of wo laid out for the weight stream.

GPU: the prepared buffer against the documented layout written out in torch
(bit-exact), and the projection bit-identical to the in-place one
(mla_output_projection / mla_output_projection_shard, which the parity tests
hold to the oracle) over batch sizes that cover the split-unit mode, the
four-block units and the direct mode, the pages' width and a tensor-parallel
column slice; one case also against the fp64 oracle directly.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_latent_attention_absorb_b200 as pkg
from sparse_latent_attention_absorb_b200 import workloads as wl

DEV = torch.device("cuda:0")


def layout_reference(wo: torch.Tensor) -> torch.Tensor:
    """The prepared layout as the header documents it, in plain torch: block
    (m, g) of 128 rows x 256 columns; inside it k-block j, 8-row group r, row
    i, 16-byte chunk q at chunk position (q ^ i)."""
    dim, k_in = wo.shape
    t = wo.reshape(dim // 128, 16, 8, k_in // 256, 4, 8, 8)  # m, r, i, g, j, q, 8 values
    i = torch.arange(8).view(1, 1, 8, 1, 1, 1)
    q = torch.arange(8).view(1, 1, 1, 1, 1, 8)
    src_q = (q ^ i).expand(dim // 128, 16, 8, k_in // 256, 4, 8)  # chunk stored at position p holds q = p ^ i
    t = torch.gather(t, 5, src_q.unsqueeze(-1).expand(*src_q.shape, 8))
    return t.permute(0, 3, 4, 1, 2, 5, 6).reshape(-1)  # m, g, j, r, i, position, values


@pytest.mark.gpu
@pytest.mark.parametrize("dim,k_in,ld", [(256, 512, 512), (384, 1024, 1536), (7168, 16384, 16384)])
def test_prepared_buffer_is_the_documented_layout(dim, k_in, ld):
    gen = torch.Generator().manual_seed(dim + k_in)
    full = torch.randint(-32768, 32767, (dim, ld), generator=gen, dtype=torch.int16).view(torch.bfloat16)
    wo = full[:, :k_in]
    got = pkg.mla_prepare_wo(full.to(DEV)[:, :k_in])
    torch.cuda.synchronize()
    # the permutation is done on the int16 view: bf16 ops may rewrite NaN payloads
    assert torch.equal(got.data.cpu().view(torch.int16), layout_reference(wo.view(torch.int16)).contiguous())


@pytest.mark.gpu
@pytest.mark.parametrize("B", [1, 3, 17, 64, 100, 300, 1000])
@pytest.mark.parametrize("dim", [128, 384, 7168])
def test_prepared_projection_equals_the_in_place_one(B, dim):
    p = wl.generate_projection(B, dim, seed=6100 + B + dim)
    x, wo = p["x"].to(DEV), p["wo"].to(DEV)
    want = pkg.mla_output_projection(x, wo)
    wp = pkg.mla_prepare_wo(wo)
    got = pkg.mla_output_projection_prepared(x, wp)
    again = pkg.mla_output_projection_prepared(x, wp)
    torch.cuda.synchronize()
    assert torch.equal(got, want)
    assert torch.equal(again, got)


@pytest.mark.gpu
@pytest.mark.parametrize("world", [2, 8])
def test_prepared_shard_equals_the_in_place_shard(world):
    B, dim = 64, wl.D_MODEL
    p = wl.generate_projection(B, dim, seed=6200 + world)
    x, wo = p["x"].to(DEV), p["wo"].to(DEV)
    k_in = 16384 // world
    for rank in (0, world - 1):
        xs = x[:, rank * k_in:(rank + 1) * k_in].contiguous()
        ws = wo[:, rank * k_in:(rank + 1) * k_in]  # strided column slice
        want = pkg.mla_output_projection_shard(xs, ws)
        got = pkg.mla_output_projection_prepared(xs, pkg.mla_prepare_wo(ws))
        torch.cuda.synchronize()
        assert torch.equal(got, want)


@pytest.mark.gpu
def test_prepared_projection_against_the_oracle():
    B, dim = 5, 1024
    p = wl.generate_projection(B, dim, seed=6301)
    got = pkg.mla_output_projection_prepared(p["x"].to(DEV), pkg.mla_prepare_wo(p["wo"].to(DEV)))
    torch.cuda.synchronize()
    want = oracle.output_projection(p["x"], p["wo"])
    g = got.double().cpu().numpy()
    tol = 2.0 ** -8 * np.abs(want) + 1e-4 * np.max(np.abs(want))
    assert np.all(np.abs(g - want) <= tol)
