"""GPU parity: the sm_100a path through the C ABI against the fp64 oracle on
the same seeded inputs.

Bounds (the decode step's stated tolerance): bf16 outputs satisfy
max|out - ref| <= 1e-2 * max|ref| + 1e-3.  Intermediate steps are checked
against the bound that their own rounding fixes (see each test).  The set of
positions with non-zero weight is checked bit-exactly by poisoning every
position that must get zero weight with NaN: the output must not change by a
single bit.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_latent_attention_absorb_b200 as pkg
from sparse_latent_attention_absorb_b200 import workloads as wl

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def out_bound(ref):
    return 1e-2 * float(np.max(np.abs(ref))) + 1e-3


def to_dev(d):
    return {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def gpu_decode(g, lse=True, d_status=None):
    B = g["q_nope"].shape[0]
    lse_out = torch.full((B, 128), float("nan"), dtype=torch.float32, device=DEV) if lse else None
    out = pkg.mla_sparse_decode(g["q_nope"], g["q_pe"], g["kv_cache"], g["pe_cache"], g["end_pos"], g["topk_idx"],
                                g["wkv_b"], g["scale"], lse_out=lse_out, d_status=d_status)
    torch.cuda.synchronize()
    return out, lse_out


def run_oracle(d, rows=None, **kw):
    return oracle.mla_sparse_decode(d["q_nope"], d["q_pe"], d["kv_cache"], d["pe_cache"], d["end_pos"],
                                    d["topk_idx"], d["wkv_b"], d["scale"], rows=rows, **kw)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_latent_attention_absorb_b200 import build
    build.build()
    pkg.load_library()


SMALL = list(wl.SMALL_WORKLOADS) + ["b1_ctx1001_top256"]


# ------------------------------------------------------------------ step a1

@pytest.mark.parametrize("B", [1, 5, 16, 64, 130])
def test_absorb_step_matches_oracle(B):
    """q_lat = bf16(q_nope . W_UK): fp32 accumulation then one bf16 rounding,
    so every element is within 2^-8 relative (+ a tiny absolute term for
    values near zero) of the exact product."""
    gen = torch.Generator().manual_seed(77 + B)
    q_nope = torch.randn((B, 128, 128), generator=gen).to(torch.bfloat16)
    wkv_b = (torch.randn((128 * 256, 512), generator=gen) * 512 ** -0.5).to(torch.bfloat16)
    q_lat = pkg.mla_absorb_q(q_nope.to(DEV), wkv_b.to(DEV))
    torch.cuda.synchronize()
    w_uk = wkv_b.double().view(128, 256, 512)[:, :128, :]
    ref = torch.einsum("bhd,hdc->bhc", q_nope.double(), w_uk).numpy()
    got = q_lat.double().cpu().numpy()
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5)


# ------------------------------------------------------------------ full path, small cases

@pytest.mark.parametrize("name", SMALL)
def test_decode_matches_oracle(name):
    d = wl.generate(name)
    g = to_dev(d)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out, lse = gpu_decode(g, d_status=status)
    ref = run_oracle(d)
    got = out.double().cpu().numpy()
    assert np.all(np.isfinite(got))
    err = np.max(np.abs(got - ref.out))
    assert err <= out_bound(ref.out), (err, out_bound(ref.out))
    # log-sum-exp: scores carry the bf16 rounding of q_lat (~1e-3 absolute)
    assert np.max(np.abs(lse.double().cpu().numpy() - ref.lse)) <= 1e-2
    assert int(status.item()) == 0


@pytest.mark.parametrize("name", ["small_b4_ctx600-2k_recent128_top400", "small_b5_ctx40-700_top333",
                                  "small_b1_ctx4096_top2048", "small_b2_ctx1500-3k_top1100"])
def test_split_outputs_combine_to_oracle_mix(name):
    """Steps a2-a6: the per-split normalised mixes and log-sum-exps, merged in
    fp64 on the host, equal the oracle's mixed latent O~ and lse."""
    d = wl.generate(name)
    g = to_dev(d)
    q_lat = pkg.mla_absorb_q(g["q_nope"], g["wkv_b"])
    o_part, lse_part = pkg.mla_sparse_attend(q_lat, g["q_pe"], g["kv_cache"], g["pe_cache"], g["end_pos"],
                                             g["topk_idx"], g["scale"])
    torch.cuda.synchronize()
    o = o_part.double().cpu().numpy()          # [B, S, H, 512]
    l = lse_part.double().cpu().numpy()        # [B, S, H]
    L = np.logaddexp.reduce(l, axis=1)         # [B, H]
    w = np.exp(l - L[:, None, :])
    merged = np.einsum("bsh,bshc->bhc", w, o)
    ref = run_oracle(d, want_o_lat=True)
    assert np.max(np.abs(L - ref.lse)) <= 1e-2
    assert np.max(np.abs(merged - ref.o_lat)) <= 1e-2 * np.max(np.abs(ref.o_lat)) + 1e-4


def test_single_split_attend_writes_the_mixed_latent():
    """Steps a2-a5 when every row is one split (B > SMs / 2): the attention
    step's output is the mixed latent O~ itself, in bf16, plus its lse."""
    name = "small_b80_ctx700_top300"
    d = wl.generate(name)
    B, K = d["topk_idx"].shape
    assert pkg.num_splits(B, K) == 1
    g = to_dev(d)
    q_lat = pkg.mla_absorb_q(g["q_nope"], g["wkv_b"])
    o_lat, lse_part = pkg.mla_sparse_attend(q_lat, g["q_pe"], g["kv_cache"], g["pe_cache"], g["end_pos"],
                                            g["topk_idx"], g["scale"])
    torch.cuda.synchronize()
    assert o_lat.dtype == torch.bfloat16 and tuple(o_lat.shape) == (B, 128, 512)
    rows = [0, 13, 41, 79]
    ref = run_oracle(d, rows=rows, want_o_lat=True)
    got = o_lat.double().cpu().numpy()[rows]
    assert np.max(np.abs(got - ref.o_lat)) <= 1e-2 * np.max(np.abs(ref.o_lat)) + 1e-4
    assert np.max(np.abs(lse_part.double().cpu().numpy()[rows, 0] - ref.lse)) <= 1e-2


@pytest.mark.parametrize("B", [7, 70])
def test_combine_step_single_split(B):
    """Steps a6-a7 with one split: O~ arrives in bf16 and goes straight into
    the W_UV product; lse passes through.  B = 70 spans two row tiles, the
    second one ragged."""
    gen = torch.Generator().manual_seed(11 + B)
    o_lat = (torch.randn((B, 128, 512), generator=gen) * 0.05).to(torch.bfloat16)
    lse_part = torch.randn((B, 1, 128), generator=gen, dtype=torch.float32) * 3
    wkv_b = (torch.randn((128 * 256, 512), generator=gen) * 512 ** -0.5).to(torch.bfloat16)
    lse_out = torch.empty((B, 128), dtype=torch.float32, device=DEV)
    out = pkg.mla_combine_value_up(o_lat.to(DEV), lse_part.to(DEV), wkv_b.to(DEV), lse_out=lse_out)
    torch.cuda.synchronize()
    w_uv = wkv_b.double().view(128, 256, 512)[:, 128:, :]
    ref = torch.einsum("bhc,hec->bhe", o_lat.double(), w_uv).numpy()
    got = out.double().cpu().numpy()
    assert np.max(np.abs(got - ref)) <= out_bound(ref)
    assert np.array_equal(lse_out.cpu().numpy(), lse_part[:, 0].numpy())


@pytest.mark.parametrize("S", [3, 40])
def test_combine_step_with_given_partials(S):
    """Steps a6-a7 alone on synthetic bf16 partials: exact LSE weights, then
    the W_UV product of the bf16-rounded mix.  S = 40 takes the split loads
    through three batches of sixteen, the last one ragged."""
    gen = torch.Generator().manual_seed(5 + S)
    B = 7  # the combine entry point accepts any split count in [1, 128]
    o_part = (torch.randn((B, S, 128, 512), generator=gen, dtype=torch.float32) * 0.05).to(torch.bfloat16)
    lse_part = torch.randn((B, S, 128), generator=gen, dtype=torch.float32) * 3
    lse_part[0, :, 5] = float("-inf")          # a row-head with no valid position
    wkv_b = (torch.randn((128 * 256, 512), generator=gen) * 512 ** -0.5).to(torch.bfloat16)
    lse_out = torch.empty((B, 128), dtype=torch.float32, device=DEV)
    out = pkg.mla_combine_value_up(o_part.to(DEV), lse_part.to(DEV), wkv_b.to(DEV), lse_out=lse_out)
    torch.cuda.synchronize()
    l = lse_part.double()
    L = torch.logsumexp(l, dim=1)
    wts = torch.exp(l - L[:, None, :]).nan_to_num(0.0)
    mixed = torch.einsum("bsh,bshc->bhc", wts, o_part.double())
    w_uv = wkv_b.double().view(128, 256, 512)[:, 128:, :]
    ref = torch.einsum("bhc,hec->bhe", mixed, w_uv).numpy()
    got = out.double().cpu().numpy()
    assert np.max(np.abs(got - ref)) <= out_bound(ref)
    assert np.all(got[0, 5] == 0.0)
    lo = lse_out.double().cpu().numpy()
    assert np.isneginf(lo[0, 5])
    fin = np.isfinite(L.numpy())
    assert np.max(np.abs(lo[fin] - L.numpy()[fin])) <= 1e-5 * (1 + np.max(np.abs(L.numpy()[fin])))


# ------------------------------------------------------------------ exact zero weights (poison)

@pytest.mark.parametrize("name", ["small_b5_ctx40-700_top333", "small_b2_ctx9000_runs6x37"])
def test_unselected_positions_get_exactly_zero_weight(name):
    d = wl.generate(name)
    g = to_dev(d)
    clean, clean_lse = gpu_decode(g)
    # NaN into every cache row that is not selected (including rows >= end_pos)
    B, S_max = d["kv_cache"].shape[:2]
    keep = torch.zeros((B, S_max), dtype=torch.bool)
    for b in range(B):
        ep = int(d["end_pos"][b])
        idx = d["topk_idx"][b]
        idx = idx[(idx >= 0) & (idx < ep)].long()
        keep[b, idx] = True
    kv = d["kv_cache"].clone()
    pe = d["pe_cache"].clone()
    kv[~keep] = float("nan")
    pe[~keep] = float("nan")
    g2 = dict(g, kv_cache=kv.to(DEV), pe_cache=pe.to(DEV))
    poisoned, poisoned_lse = gpu_decode(g2)
    assert torch.equal(clean.view(torch.int16), poisoned.view(torch.int16))
    assert torch.equal(clean_lse, poisoned_lse)
    assert torch.isfinite(clean.float()).all()


def test_index_order_and_padding_placement_do_not_matter():
    d = wl.generate("small_b4_ctx600-2k_recent128_top400")
    g = to_dev(d)
    base, _ = gpu_decode(g)
    gen = torch.Generator().manual_seed(3)
    idx = d["topk_idx"].clone()
    for b in range(idx.shape[0]):
        idx[b] = idx[b, torch.randperm(idx.shape[1], generator=gen)]
    shuffled, _ = gpu_decode(dict(g, topk_idx=idx.to(DEV)))
    ref = run_oracle(d)
    assert np.max(np.abs(shuffled.double().cpu().numpy() - ref.out)) <= out_bound(ref.out)
    assert np.max(np.abs(shuffled.double().cpu().numpy() - base.double().cpu().numpy())) <= out_bound(ref.out)


def test_rows_without_valid_index_and_out_of_range_entries():
    d = wl.generate("small_b5_ctx40-700_top333")
    idx = d["topk_idx"].clone()
    idx[1] = -1                                       # nothing selected
    idx[2, :5] = torch.tensor([-7, 10 ** 6, int(d["end_pos"][2]), 704, -1], dtype=torch.int32)
    d2 = dict(d, topk_idx=idx)
    out, lse = gpu_decode(to_dev(d2))
    ref = run_oracle(d2)
    got = out.double().cpu().numpy()
    assert np.all(got[1] == 0.0)
    assert np.all(np.isneginf(lse.cpu().numpy()[1]))
    assert np.max(np.abs(got - ref.out)) <= out_bound(ref.out)


def test_single_selected_position_closed_form():
    """|T_b| = 1: out[b,h] = W_UV[h] . kv[b,t] whatever the query (up to bf16
    rounding of the mixed latent, which here is the cached row itself)."""
    d = wl.generate("small_b2_ctx300_top100")
    idx = torch.full_like(d["topk_idx"], -1)
    idx[0, 37] = 123
    idx[1, 0] = 0
    d2 = dict(d, topk_idx=idx)
    out, _ = gpu_decode(to_dev(d2))
    w_uv = d["wkv_b"].double().view(128, 256, 512)[:, 128:, :]
    for b, t in ((0, 123), (1, 0)):
        ref = torch.einsum("hec,c->he", w_uv, d["kv_cache"][b, t].double()).numpy()
        got = out[b].double().cpu().numpy()
        assert np.max(np.abs(got - ref)) <= out_bound(ref)


def test_repeated_calls_are_deterministic():
    d = wl.generate("small_b3_ctx1001_top256")
    g = to_dev(d)
    a, la = gpu_decode(g)
    b, lb = gpu_decode(g)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16)) and torch.equal(la, lb)


def test_workspace_too_small_is_rejected():
    d = wl.generate("small_b2_ctx300_top100")
    g = to_dev(d)
    B, K, S = d["q_nope"].shape[0], d["topk_idx"].shape[1], d["kv_cache"].shape[1]
    ws = torch.empty(pkg.workspace_size(B, K, S) - 256, dtype=torch.uint8, device=DEV)
    with pytest.raises(pkg.MLAError) as e:
        pkg.mla_sparse_decode(g["q_nope"], g["q_pe"], g["kv_cache"], g["pe_cache"], g["end_pos"], g["topk_idx"],
                              g["wkv_b"], g["scale"], workspace=ws)
    assert e.value.code == 2


# ------------------------------------------------------------------ full-size workloads, sampled rows

FULL = ["b8_ctx4096_top2048", "b32_ctx2k-8k_recent512_top2048", "b64_ctx1k-32k_top2048",
        "b16_ctx131072_runs32x64", "b16_ctx8192_dense"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_workloads_sampled_rows(name):
    """The benchmark's launch configuration at the full sizes; the oracle
    recomputes a sample of batch rows (all 128 heads each)."""
    d = wl.generate(name)
    g = to_dev(d)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out, lse = gpu_decode(g, d_status=status)
    B = d["q_nope"].shape[0]
    rows = sorted({0, B - 1, B // 2, (7 * B) // 11})
    ref = run_oracle(d, rows=rows)
    got = out.double().cpu().numpy()[rows]
    assert np.all(np.isfinite(out.float().cpu().numpy()))
    assert np.max(np.abs(got - ref.out)) <= out_bound(ref.out)
    assert np.max(np.abs(lse.double().cpu().numpy()[rows] - ref.lse)) <= 1e-2
    assert int(status.item()) == 0
    del g
    torch.cuda.empty_cache()


def test_more_rows_than_tiles_and_clusters():
    """B = 150 rows of one split each: two row tiles in the absorption kernel,
    more 2-CTA clusters than the GPU holds at once (a second wave), and three
    row tiles in the value-up kernel, the last one ragged (22 rows, the rest
    read as zero by TMA)."""
    w = wl.Workload("t_b150_ctx200-300_top100", 150, 300, (200, 300), 100, "uniform", 3001)
    d = wl.generate(w)
    assert pkg.num_splits(150, 100) == 1
    out, lse = gpu_decode(to_dev(d))
    ref = run_oracle(d)
    got = out.double().cpu().numpy()
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(got - ref.out)) <= out_bound(ref.out)
    assert np.max(np.abs(lse.double().cpu().numpy() - ref.lse)) <= 1e-2


def test_online_softmax_rescales_when_scores_grow_along_the_tiles():
    """Scores that grow with position, visited in ascending order: the running
    maximum jumps by more than 2^8 on nearly every tile, so O is rescaled in
    place many times.  The result must still match the oracle."""
    d = wl.generate("small_b80_ctx700_top300")
    B, S = d["q_nope"].shape[0], d["kv_cache"].shape[1]
    pos = torch.arange(S, dtype=torch.float32)
    pe = (pos[None, :, None] * 0.02).expand(B, S, 64).to(torch.bfloat16).contiguous()
    q_pe = torch.ones_like(d["q_pe"])
    idx = d["topk_idx"].clone()
    for b in range(B):
        v = idx[b][idx[b] >= 0]
        idx[b] = -1
        idx[b, : v.numel()] = torch.sort(v).values
    d2 = dict(d, pe_cache=pe, q_pe=q_pe, topk_idx=idx)
    out, lse = gpu_decode(to_dev(d2))
    rows = [0, 17, 42, 79]
    ref = run_oracle(d2, rows=rows)
    got = out.double().cpu().numpy()[rows]
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(got - ref.out)) <= out_bound(ref.out)
    assert np.max(np.abs(lse.double().cpu().numpy()[rows] - ref.lse)) <= 1e-2


# ------------------------------------------------------------------ output projection (page "Attention update")

def proj_bound(ref):
    """bf16 of an fp32 sum: one bf16 rounding (half an ulp is 2^-9 relative;
    2^-8 allowed) plus fp32 accumulation over 16384 products in an order the
    oracle does not fix (bounded by 1e-4 of the largest output)."""
    return 2.0 ** -8 * np.abs(ref) + 1e-4 * float(np.max(np.abs(ref)))


@pytest.mark.parametrize("B,dim", [(1, 128), (3, 384), (17, 1024), (64, 7168), (100, 2048), (300, 256),
                                   (1000, 7168)])
def test_output_projection_matches_oracle(B, dim):
    """delta = x . wo^T.  Covers: fewer tiles than SMs (work split unit by
    unit, partials reduced in a fixed order; B=1, dim=128 spreads one tile
    over all SMs), two batch tiles (B=300), and one CTA per tile writing
    bf16 directly (B=1000 at the pages' width: 4 x 56 tiles)."""
    d = wl.generate_projection(B, dim, seed=3000 + B)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    delta = pkg.mla_output_projection(d["x"].to(DEV), d["wo"].to(DEV), d_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rows = list(range(B)) if B <= 17 else sorted({0, 1, B // 2, B - 2, B - 1})
    ref = oracle.output_projection(d["x"], d["wo"], rows=rows)
    got = delta.double().cpu().numpy()[rows]
    assert np.all(np.abs(got - ref) <= proj_bound(ref))


def test_output_projection_is_deterministic():
    d = wl.generate_projection(64, 1024, seed=3100)
    x, wo = d["x"].to(DEV), d["wo"].to(DEV)
    a = pkg.mla_output_projection(x, wo)
    b = pkg.mla_output_projection(x, wo)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("name", ["small_b5_ctx40-700_top333", "b1_ctx1001_top256"])
def test_decode_project_matches_oracle_chain(name):
    """The fused call equals the two separate calls bit for bit, and the
    oracle's decode followed by its projection within the decode step's
    tolerance (the decode's rounding passes through wo, whose rows have unit
    norm)."""
    d = wl.generate(name)
    g = to_dev(d)
    B = d["q_nope"].shape[0]
    wo_cpu = wl.generate_projection(1, wl.D_MODEL, seed=3200)["wo"]
    wo = wo_cpu.to(DEV)
    delta = pkg.mla_sparse_decode_project(g["q_nope"], g["q_pe"], g["kv_cache"], g["pe_cache"], g["end_pos"],
                                          g["topk_idx"], g["wkv_b"], g["scale"], wo)
    out, _ = gpu_decode(g, lse=False)
    delta2 = pkg.mla_output_projection(out, wo)
    torch.cuda.synchronize()
    assert torch.equal(delta, delta2)
    ref_out = run_oracle(d).out                                   # fp64 [B, 128, 128]
    ref = oracle.output_projection(ref_out, wo_cpu.double().numpy())
    got = delta.double().cpu().numpy()
    assert got.shape == (B, wl.D_MODEL)
    assert np.max(np.abs(got - ref)) <= out_bound(ref)


# ------------------------------------------------------------------ sparse prefill (page "Queries", prefill mode)

def _prefill_dev(d):
    return {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


@pytest.mark.parametrize("B,seqlen,K", [(2, 300, 128), (1, 700, 256)])
def test_prefill_matches_oracle(B, seqlen, K):
    """One row per query position, each reading its sequence's latents up to
    its causal bound (rows with fewer than K valid positions included)."""
    d = wl.generate_prefill(B, seqlen, K, seed=2200 + seqlen)
    g = _prefill_dev(d)
    R = B * seqlen
    lse = torch.full((R, 128), float("nan"), dtype=torch.float32, device=DEV)
    out = pkg.mla_sparse_prefill(g["q_nope"], g["q_pe"], g["kv_cache"], g["pe_cache"], g["cache_slot"], g["end_pos"],
                                 g["topk_idx"], g["wkv_b"], g["scale"], lse_out=lse)
    torch.cuda.synchronize()
    rows = sorted({0, 1, 2, K - 2, K - 1, K, K + 1, seqlen - 1, seqlen, R // 2, R - 1} & set(range(R)))
    ref = oracle.mla_sparse_decode(d["q_nope"], d["q_pe"], d["kv_cache"], d["pe_cache"], d["end_pos"],
                                   d["topk_idx"], d["wkv_b"], d["scale"], rows=rows, cache_slot=d["cache_slot"])
    got = out.double().cpu().numpy()[rows]
    assert np.max(np.abs(got - ref.out)) <= out_bound(ref.out)
    assert np.max(np.abs(lse.double().cpu().numpy()[rows] - ref.lse)) <= 1e-2


def test_prefill_with_identity_slots_equals_decode():
    d = wl.generate("small_b5_ctx40-700_top333")
    g = to_dev(d)
    B = d["q_nope"].shape[0]
    slots = torch.arange(B, dtype=torch.int32, device=DEV)
    out_p = pkg.mla_sparse_prefill(g["q_nope"], g["q_pe"], g["kv_cache"], g["pe_cache"], slots, g["end_pos"],
                                   g["topk_idx"], g["wkv_b"], g["scale"])
    out_d, _ = gpu_decode(g, lse=False)
    assert torch.equal(out_p, out_d)


def test_prefill_rows_with_an_out_of_range_slot_are_empty():
    d = wl.generate_prefill(2, 70, 32, seed=2300)
    g = _prefill_dev(d)
    R = 140
    lse = torch.empty((R, 128), dtype=torch.float32, device=DEV)
    good = pkg.mla_sparse_prefill(g["q_nope"], g["q_pe"], g["kv_cache"], g["pe_cache"], g["cache_slot"], g["end_pos"],
                                  g["topk_idx"], g["wkv_b"], g["scale"]).clone()
    slots = g["cache_slot"].clone()
    slots[5], slots[100] = 2, -7
    out = pkg.mla_sparse_prefill(g["q_nope"], g["q_pe"], g["kv_cache"], g["pe_cache"], slots, g["end_pos"],
                                 g["topk_idx"], g["wkv_b"], g["scale"], lse_out=lse)
    torch.cuda.synchronize()
    for r in (5, 100):
        assert torch.all(out[r] == 0) and torch.all(torch.isneginf(lse[r]))
    keep = [r for r in range(R) if r not in (5, 100)]
    assert torch.equal(out[keep], good[keep])
