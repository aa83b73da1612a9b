"""Pins for the fp64 oracle (CPU only).

The pages print no numeric worked example, so the oracle is pinned to what
the pages and the mathematics fix:
  (a) absorption: the non-absorbed "MHA prefill" form and the identity
      A(c W_UV) = (A c) W_UV ("Apply value weights");
  (b) softmax: rows sum to 1, masked positions get weight exactly 0
      ("Softmax"; the -inf index mask of the decode excerpt);
  (c) dense: with every position selected the result is plain attention,
      computed by torch's scaled_dot_product_attention in float64;
  (d) brute force: every non-empty mask on tiny inputs against the decode
      excerpt's einsums run literally in torch float64;
  plus closed forms (one selected key; zero query) and set semantics of the
  index list (order, duplicates, padding).
The per-row cache slot (one row per query position of a sequence) is pinned
by the page's "MHA prefill" excerpt (page "Queries") run as written in torch
float64 with the causal and index masks.
The output projection (page "Attention update") is pinned by a hand-derived
case, basis vectors (a unit input picks one column of wo), linearity, BLAS
float64 matmul, and the page's ``wo(x.flatten(2))`` in torch float64.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from tests.oracle_refs import (nonabsorbed, prefill_transcript, transcript, transcript_projection, to_f64,
                               valid_set)
from sparse_latent_attention_absorb_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_case(rng, B, H, Dn, Dr, Dl, Dv, S_max, K, ep_lo=None, pad=True):
    """Random fp64 inputs with distinct shuffled indices, -1 padded."""
    q_nope = rng.standard_normal((B, H, Dn))
    q_pe = rng.standard_normal((B, H, Dr))
    kv = rng.standard_normal((B, S_max, Dl))
    pe = rng.standard_normal((B, S_max, Dr))
    wkv_b = rng.standard_normal((H * (Dn + Dv), Dl)) / math.sqrt(Dl)
    lo = S_max if ep_lo is None else ep_lo
    end_pos = rng.integers(lo, S_max + 1, size=B).astype(np.int32)
    idx = np.full((B, K), -1, np.int32)
    for b in range(B):
        k = min(K, int(end_pos[b])) if pad else K
        sel = rng.permutation(int(end_pos[b]))[:k]
        idx[b, :len(sel)] = sel
    scale = (Dn + Dr) ** -0.5
    return dict(q_nope=q_nope, q_pe=q_pe, kv_cache=kv, pe_cache=pe, wkv_b=wkv_b,
                end_pos=end_pos, topk_idx=idx, scale=scale)


def run(case, **kw):
    return oracle.mla_sparse_decode(case["q_nope"], case["q_pe"], case["kv_cache"], case["pe_cache"],
                                    case["end_pos"], case["topk_idx"], case["wkv_b"], case["scale"], **kw)


def rel_err(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


# ---------------------------------------------------------------- (a) absorption

@pytest.mark.parametrize("dims", [
    dict(B=2, H=3, Dn=4, Dr=2, Dl=5, Dv=3, S_max=9, K=6, ep_lo=4),
    dict(B=3, H=8, Dn=16, Dr=8, Dl=32, Dv=12, S_max=70, K=40, ep_lo=20),
    dict(B=1, H=128, Dn=128, Dr=64, Dl=512, Dv=128, S_max=300, K=64),
])
def test_absorbed_equals_nonabsorbed_prefill_form(dims):
    rng = np.random.default_rng(1)
    case = rand_case(rng, **dims)
    res = run(case)
    ref = nonabsorbed(case["q_nope"], case["q_pe"], case["kv_cache"], case["pe_cache"],
                      case["wkv_b"], case["end_pos"], case["topk_idx"], case["scale"], Dv=dims["Dv"])
    assert rel_err(res.out, ref) <= 1e-10


def test_value_up_identity_mix_then_project():
    """A (c W_UV) == (A c) W_UV: the oracle mixes latents first; projecting
    every selected latent first and mixing after must agree."""
    rng = np.random.default_rng(2)
    B, H, Dn, Dr, Dl, Dv, S = 2, 4, 6, 2, 10, 5, 30
    case = rand_case(rng, B, H, Dn, Dr, Dl, Dv, S, 12, ep_lo=15)
    res = run(case, want_o_lat=True, want_weights=True)
    w_uv = case["wkv_b"].reshape(H, Dn + Dv, Dl)[:, Dn:, :]
    for b in range(B):
        for h in range(H):
            A = res.w_full[b, h]                            # weights over positions
            projected_first = A @ (case["kv_cache"][b] @ w_uv[h].T)
            mixed_first = (A @ case["kv_cache"][b]) @ w_uv[h].T
            np.testing.assert_allclose(projected_first, mixed_first, rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(res.out[b, h], mixed_first, rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(res.o_lat[b, h], A @ case["kv_cache"][b], rtol=1e-12, atol=1e-14)


def test_q_lat_is_the_absorbed_query():
    rng = np.random.default_rng(3)
    H, Dn, Dv, Dl = 5, 7, 3, 9
    case = rand_case(rng, 2, H, Dn, 2, Dl, Dv, 8, 4)
    res = run(case, want_q_lat=True)
    w_uk = case["wkv_b"].reshape(H, Dn + Dv, Dl)[:, :Dn, :]
    ref = np.einsum("bhd,hdc->bhc", case["q_nope"], w_uk)
    np.testing.assert_allclose(res.q_lat, ref, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- (b) softmax

def test_softmax_rows_sum_to_one_and_mask_is_exact_zero():
    rng = np.random.default_rng(4)
    B, H, S = 3, 6, 50
    case = rand_case(rng, B, H, 8, 4, 16, 8, S, 20, ep_lo=10)
    res = run(case, want_weights=True)
    for b in range(B):
        T = set(valid_set(case["topk_idx"][b], int(case["end_pos"][b])))
        for h in range(H):
            w = res.w_full[b, h]
            assert abs(w.sum() - 1.0) <= 1e-12
            for t in range(S):
                if t in T:
                    assert w[t] > 0.0
                else:
                    assert w[t] == 0.0          # exp(-inf) = 0, exactly


def test_lse_matches_its_definition():
    rng = np.random.default_rng(5)
    H, Dn, Dr, Dl, Dv = 3, 4, 2, 6, 3
    case = rand_case(rng, 2, H, Dn, Dr, Dl, Dv, 12, 7)
    res = run(case)
    w_uk = case["wkv_b"].reshape(H, Dn + Dv, Dl)[:, :Dn, :]
    for b in range(2):
        T = valid_set(case["topk_idx"][b], int(case["end_pos"][b]))
        for h in range(H):
            ql = case["q_nope"][b, h] @ w_uk[h]
            s = [(ql @ case["kv_cache"][b, t] + case["q_pe"][b, h] @ case["pe_cache"][b, t]) * case["scale"]
                 for t in T]
            assert abs(res.lse[b, h] - math.log(sum(math.exp(x) for x in s))) <= 1e-12


# ---------------------------------------------------------------- (c) dense

@pytest.mark.parametrize("H,Dn,Dr,Dl,Dv,S", [(4, 8, 4, 16, 8, 33), (128, 128, 64, 512, 128, 96)])
def test_dense_selection_equals_library_sdpa(H, Dn, Dr, Dl, Dv, S):
    """With T_b = [0, end_pos) the masked softmax is plain attention: compare
    with torch.nn.functional.scaled_dot_product_attention in float64 on the
    up-projected (non-absorbed) q, k, v."""
    rng = np.random.default_rng(6)
    B = 2
    case = rand_case(rng, B, H, Dn, Dr, Dl, Dv, S, S)
    case["end_pos"][:] = S
    case["topk_idx"][:] = np.stack([rng.permutation(S) for _ in range(B)])
    res = run(case)
    wb = case["wkv_b"].reshape(H, Dn + Dv, Dl)
    for b in range(B):
        c = torch.tensor(case["kv_cache"][b])
        k_nope = torch.einsum("hdc,tc->htd", torch.tensor(wb[:, :Dn]), c)
        v = torch.einsum("hdc,tc->htd", torch.tensor(wb[:, Dn:]), c)
        k = torch.cat([k_nope, torch.tensor(case["pe_cache"][b]).expand(H, S, Dr)], dim=-1)
        q = torch.cat([torch.tensor(case["q_nope"][b]), torch.tensor(case["q_pe"][b])], dim=-1)[:, None, :]
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=case["scale"])
        np.testing.assert_allclose(res.out[b], o[:, 0, :].numpy(), rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- (d) brute force

def test_bruteforce_every_mask_tiny_against_transcript():
    """H=2, Dn=4, Dr=2, Dl=3, Dv=2, end_pos <= 5: every non-empty subset of
    positions as the top-k set, against the decode excerpt run literally."""
    rng = np.random.default_rng(7)
    H, Dn, Dr, Dl, Dv = 2, 4, 2, 3, 2
    n_checked = 0
    for ep in range(1, 6):
        base = rand_case(rng, 1, H, Dn, Dr, Dl, Dv, ep, ep)
        base["end_pos"][:] = ep
        for r in range(1, ep + 1):
            for subset in itertools.combinations(range(ep), r):
                case = dict(base)
                idx = np.full((1, ep), -1, np.int32)
                idx[0, :r] = rng.permutation(np.array(subset, np.int32))
                case["topk_idx"] = idx
                res = run(case)
                ref = transcript(case["q_nope"], case["q_pe"], case["kv_cache"], case["pe_cache"],
                                 case["wkv_b"], case["end_pos"], idx, case["scale"], Dv=Dv)
                assert rel_err(res.out, ref) <= 1e-12, (ep, subset)
                n_checked += 1
    assert n_checked == 1 + 3 + 7 + 15 + 31


def test_transcript_agrees_on_real_dims_bf16_inputs():
    """The excerpt's einsums on a reduced copy of the pages' workload, bf16
    inputs widened exactly."""
    d = wl.generate("small_b2_ctx300_top100")
    res = oracle.mla_sparse_decode(d["q_nope"], d["q_pe"], d["kv_cache"], d["pe_cache"], d["end_pos"],
                                   d["topk_idx"], d["wkv_b"], d["scale"])
    ref = transcript(d["q_nope"], d["q_pe"], d["kv_cache"], d["pe_cache"], d["wkv_b"], d["end_pos"].numpy(),
                     d["topk_idx"].numpy(), d["scale"])
    assert rel_err(res.out, ref) <= 1e-12


# ---------------------------------------------------------------- closed forms

def test_single_selected_key_gives_its_projected_value():
    """|T_b| = 1: the softmax weight is 1 whatever q is, so the output is
    W_UV[h] applied to that one cached latent."""
    rng = np.random.default_rng(8)
    H, Dn, Dr, Dl, Dv, S = 3, 4, 2, 6, 5, 10
    case = rand_case(rng, 2, H, Dn, Dr, Dl, Dv, S, 3)
    case["topk_idx"][:] = -1
    case["topk_idx"][0, 1] = 7
    case["topk_idx"][1, 2] = 0
    case["q_nope"] *= 100.0                      # irrelevant to the result
    res = run(case, want_weights=True)
    w_uv = case["wkv_b"].reshape(H, Dn + Dv, Dl)[:, Dn:, :]
    for b, t in ((0, 7), (1, 0)):
        for h in range(H):
            np.testing.assert_allclose(res.out[b, h], w_uv[h] @ case["kv_cache"][b, t], rtol=1e-13, atol=1e-14)
            assert res.w_full[b, h, t] == 1.0


@pytest.mark.parametrize("zero", ["query", "scale"])
def test_zero_scores_give_mean_of_selected_values(zero):
    rng = np.random.default_rng(9)
    H, Dn, Dr, Dl, Dv, S = 3, 4, 2, 6, 5, 20
    case = rand_case(rng, 2, H, Dn, Dr, Dl, Dv, S, 9, ep_lo=12)
    if zero == "query":
        case["q_nope"][:] = 0.0
        case["q_pe"][:] = 0.0
    else:
        case["scale"] = 0.0
    res = run(case)
    w_uv = case["wkv_b"].reshape(H, Dn + Dv, Dl)[:, Dn:, :]
    for b in range(2):
        T = valid_set(case["topk_idx"][b], int(case["end_pos"][b]))
        mean = case["kv_cache"][b, T].mean(axis=0)
        for h in range(H):
            np.testing.assert_allclose(res.out[b, h], w_uv[h] @ mean, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(res.lse[b], math.log(len(T)), rtol=1e-13)


def test_two_keys_hand_derived():
    """H = Dn = Dr = Dl = Dv = 1, W_UK = 1, W_UV = 2, q_nope = 1, q_pe = 0.5,
    latents c = (0, ln 3), rotary keys (0, 0), scale 1: scores (0, ln 3),
    weights (1/4, 3/4), mixed latent (3/4) ln 3, output (3/2) ln 3,
    lse = ln 4."""
    case = dict(q_nope=np.ones((1, 1, 1)), q_pe=np.full((1, 1, 1), 0.5),
                kv_cache=np.array([[[0.0], [math.log(3.0)]]]), pe_cache=np.zeros((1, 2, 1)),
                wkv_b=np.array([[1.0], [2.0]]), end_pos=np.array([2], np.int32),
                topk_idx=np.array([[1, 0]], np.int32), scale=1.0)
    res = run(case, want_weights=True, want_o_lat=True)
    assert res.w_full[0, 0].tolist() == pytest.approx([0.25, 0.75], abs=1e-15)
    assert res.o_lat[0, 0, 0] == pytest.approx(0.75 * math.log(3.0), abs=1e-15)
    assert res.out[0, 0, 0] == pytest.approx(1.5 * math.log(3.0), abs=1e-15)
    assert res.lse[0, 0] == pytest.approx(math.log(4.0), abs=1e-15)


def test_rotary_term_and_scale_placement_hand_derived():
    """Scores come from the latent and rotary parts summed, then scaled:
    q_lat = 2 (q_nope 1, W_UK 2), c = (1, 0), q_pe = 1, k^R = (0, ln 9),
    scale 1/2: s = ((2*1 + 0), (0 + ln 9)) / 2 = (1, ln 3); weights
    e/(e+3), 3/(e+3); with W_UV = 1 the output is the mixed latent e/(e+3)."""
    case = dict(q_nope=np.ones((1, 1, 1)), q_pe=np.ones((1, 1, 1)),
                kv_cache=np.array([[[1.0], [0.0]]]), pe_cache=np.array([[[0.0], [math.log(9.0)]]]),
                wkv_b=np.array([[2.0], [1.0]]), end_pos=np.array([2], np.int32),
                topk_idx=np.array([[0, 1]], np.int32), scale=0.5)
    res = run(case)
    e = math.e
    assert res.out[0, 0, 0] == pytest.approx(e / (e + 3.0), abs=1e-15)
    assert res.lse[0, 0] == pytest.approx(math.log(e + 3.0), abs=1e-15)


# ---------------------------------------------------------------- index-set semantics

def test_index_order_duplicates_and_padding_do_not_matter():
    rng = np.random.default_rng(10)
    case = rand_case(rng, 2, 4, 8, 4, 16, 8, 40, 15, ep_lo=30)
    base = run(case).out
    # order
    c2 = dict(case, topk_idx=case["topk_idx"][:, ::-1].copy())
    assert np.array_equal(run(c2).out, base)
    # duplicates and out-of-range entries (negative, >= end_pos, >= S_max)
    extra = np.concatenate([case["topk_idx"], case["topk_idx"][:, :5],
                            np.full((2, 3), -7, np.int32),
                            np.stack([case["end_pos"], case["end_pos"] + 3, np.full(2, 10 ** 6)], 1).astype(np.int32)],
                           axis=1)
    c3 = dict(case, topk_idx=extra)
    assert np.array_equal(run(c3).out, base)


def test_row_without_valid_index_gives_zero_and_neg_inf_lse():
    rng = np.random.default_rng(11)
    case = rand_case(rng, 2, 3, 4, 2, 6, 3, 10, 4)
    case["topk_idx"][1] = -1
    res = run(case)
    assert np.all(res.out[1] == 0.0)
    assert np.all(np.isneginf(res.lse[1]))
    assert np.all(np.isfinite(res.out[0]))


def test_row_subset_selection_matches_full_run():
    d = wl.generate("small_b5_ctx40-700_top333")
    args = (d["q_nope"], d["q_pe"], d["kv_cache"], d["pe_cache"], d["end_pos"], d["topk_idx"], d["wkv_b"], d["scale"])
    full = oracle.mla_sparse_decode(*args)
    part = oracle.mla_sparse_decode(*args, rows=[4, 1])
    assert np.array_equal(part.out[0], full.out[4])
    assert np.array_equal(part.out[1], full.out[1])


# ---------------------------------------------------------------- golden fixtures

def test_page_shapes_fixture():
    """Dimensions the pages print, against the workload generator."""
    with open(os.path.join(GOLDEN, "page_shapes.json")) as f:
        g = json.load(f)
    assert g["heads"] == wl.H
    assert g["latent_plus_rotary"] == wl.D_LAT + wl.D_ROPE
    assert g["content_plus_rotary"] == wl.D_NOPE + wl.D_ROPE
    assert g["kv_latent"] == wl.D_LAT and g["value"] == wl.D_V
    assert g["cached_positions_example"] == wl.WORKLOADS["b1_ctx1001_top256"].end_pos[0]
    assert wl.SCALE == pytest.approx(g["content_plus_rotary"] ** -0.5, rel=1e-7)
    assert g["model_width"] == wl.D_MODEL
    assert g["wo_inputs"] == g["heads"] * g["value"] == wl.H * wl.D_V
    d = wl.generate_projection(2, dim=256)
    assert tuple(d["x"].shape) == (2, g["wo_inputs"]) and tuple(d["wo"].shape) == (256, g["wo_inputs"])


def test_regression_fixture():
    """Stored oracle outputs (written by tests/golden/make_golden.py, which
    calls only the oracle) on a seeded tiny case: guards against accidental
    changes of the oracle's arithmetic."""
    with open(os.path.join(GOLDEN, "oracle_tiny_regression.json")) as f:
        g = json.load(f)
    from tests.golden.make_golden import tiny_case
    case = tiny_case()
    res = run(case)
    np.testing.assert_allclose(res.out.reshape(-1), np.array(g["out"]), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(res.lse.reshape(-1), np.array(g["lse"]), rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- output projection

def test_projection_hand_derived():
    x = np.array([[1.0, 2.0, 3.0], [0.5, -1.0, 0.0]])
    wo = np.array([[1.0, 0.0, 0.0], [0.0, 1.0, 1.0], [2.0, -1.0, 0.5]])
    # row 0: (1, 2 + 3, 2 - 2 + 1.5); row 1: (0.5, -1, 1 + 1 + 0)
    np.testing.assert_array_equal(oracle.output_projection(x, wo), [[1.0, 5.0, 1.5], [0.5, -1.0, 2.0]])


def test_projection_unit_inputs_pick_columns_of_wo():
    rng = np.random.default_rng(11)
    n_in, dim = 64, 40
    wo = rng.standard_normal((dim, n_in))
    ks = [0, 7, 31, 63]
    x = np.zeros((len(ks), n_in))
    for r, k in enumerate(ks):
        x[r, k] = 1.0
    got = oracle.output_projection(x, wo)
    for r, k in enumerate(ks):
        np.testing.assert_array_equal(got[r], wo[:, k])


def test_projection_is_linear():
    rng = np.random.default_rng(12)
    n_in, dim = 96, 33
    wo = rng.standard_normal((dim, n_in))
    x1, x2 = rng.standard_normal((3, n_in)), rng.standard_normal((3, n_in))
    a = 0.75
    lhs = oracle.output_projection(a * x1 + x2, wo)
    rhs = a * oracle.output_projection(x1, wo) + oracle.output_projection(x2, wo)
    assert rel_err(lhs, rhs) < 1e-13


def test_projection_matches_blas_and_page_transcript_at_real_width():
    """bf16 inputs of the real shapes (x [B,128,128] flattened per row, wo
    [dim,16384]), widened exactly: BLAS float64 matmul and the page's
    wo(x.flatten(2)) agree with the oracle."""
    d = wl.generate_projection(3, dim=256, seed=17)
    x3 = d["x"].view(3, wl.H, wl.D_V)
    got = oracle.output_projection(x3, d["wo"])
    blas = to_f64(d["x"]) @ to_f64(d["wo"]).T
    assert rel_err(got, blas) < 1e-12
    assert rel_err(got, transcript_projection(x3, d["wo"])) < 1e-12
    # the flattening is per row, head-major: k = 128 h + e
    assert got[1, 5] == pytest.approx(float(sum(to_f64(x3)[1, h, e] * to_f64(d["wo"])[5, 128 * h + e]
                                                for h in range(wl.H) for e in range(wl.D_V))), rel=1e-12)


def test_projection_row_subset_matches_full_run():
    d = wl.generate_projection(5, dim=128, seed=18)
    full = oracle.output_projection(d["x"], d["wo"])
    part = oracle.output_projection(d["x"], d["wo"], rows=[4, 0])
    np.testing.assert_array_equal(part, full[[4, 0]])
    with pytest.raises(RuntimeError):
        oracle.output_projection(d["x"], d["wo"], rows=[5])


# ---------------------------------------------------------------- prefill rows (page "Queries")

def _prefill_case(rng, bsz, seqlen, K, H, Dn, Dr, Dl, Dv):
    q_nope = rng.standard_normal((bsz, seqlen, H, Dn))
    q_pe = rng.standard_normal((bsz, seqlen, H, Dr))
    kv = rng.standard_normal((bsz, seqlen, Dl))
    k_pe = rng.standard_normal((bsz, seqlen, Dr))
    wkv_b = rng.standard_normal((H * (Dn + Dv), Dl)) / math.sqrt(Dl)
    # the indexer returns K positions of the chunk for every query; with its
    # scores causally masked the query's own position is among them, later
    # ones may follow (the causal mask removes them)
    topk = np.zeros((bsz, seqlen, K), np.int64)
    for b in range(bsz):
        for s_ in range(seqlen):
            others = [t for t in rng.permutation(seqlen) if t != s_][:K - 1]
            topk[b, s_] = [s_] + others
    return q_nope, q_pe, kv, k_pe, wkv_b, topk.astype(np.int32)


def _prefill_oracle(q_nope, q_pe, kv, k_pe, wkv_b, topk, scale, **kw):
    bsz, seqlen, H = q_nope.shape[:3]
    R = bsz * seqlen
    slot = np.repeat(np.arange(bsz, dtype=np.int32), seqlen)
    end_pos = np.tile(np.arange(1, seqlen + 1, dtype=np.int32), bsz)
    return oracle.mla_sparse_decode(q_nope.reshape(R, H, -1), q_pe.reshape(R, H, -1), kv, k_pe, end_pos,
                                    topk.reshape(R, -1), wkv_b, scale, cache_slot=slot, **kw)


@pytest.mark.parametrize("dims", [dict(H=2, Dn=4, Dr=2, Dl=6, Dv=3, bsz=2, seqlen=7, K=3),
                                  dict(H=128, Dn=128, Dr=64, Dl=512, Dv=128, bsz=1, seqlen=10, K=4)])
def test_prefill_rows_equal_page_prefill_excerpt(dims):
    rng = np.random.default_rng(21)
    d = dict(dims)
    bsz, seqlen, K = d.pop("bsz"), d.pop("seqlen"), d.pop("K")
    case = _prefill_case(rng, bsz, seqlen, K, **d)
    scale = (d["Dn"] + d["Dr"]) ** -0.5
    got = _prefill_oracle(*case, scale).out.reshape(bsz, seqlen, d["H"], d["Dv"])
    ref = prefill_transcript(*case, scale, d["Dv"])
    assert rel_err(got, ref) < 1e-10


def test_prefill_slot_out_of_range_gives_an_empty_row():
    rng = np.random.default_rng(22)
    q_nope, q_pe, kv, k_pe, wkv_b, topk = _prefill_case(rng, 2, 5, 3, H=2, Dn=4, Dr=2, Dl=6, Dv=3)
    R = 10
    slot = np.repeat(np.arange(2, dtype=np.int32), 5)
    slot[3], slot[7] = 2, -1
    end_pos = np.tile(np.arange(1, 6, dtype=np.int32), 2)
    res = oracle.mla_sparse_decode(q_nope.reshape(R, 2, 4), q_pe.reshape(R, 2, 2), kv, k_pe, end_pos,
                                   topk.reshape(R, 3), wkv_b, 0.4, cache_slot=slot)
    for r in (3, 7):
        assert np.all(res.out[r] == 0.0) and np.all(res.lse[r] == -np.inf)
    good = [r for r in range(R) if r not in (3, 7)]
    ref = _prefill_oracle(q_nope, q_pe, kv, k_pe, wkv_b, topk, 0.4)
    np.testing.assert_array_equal(res.out[good], ref.out[good])


def test_next_rows_regression_fixture():
    """Stored oracle outputs for per-row cache slots (prefill rows) and the
    output projection (written by tests/golden/make_golden.py, which calls
    only the oracle): guards against accidental changes of their arithmetic."""
    with open(os.path.join(GOLDEN, "oracle_next_rows_regression.json")) as f:
        g = json.load(f)
    from tests.golden.make_golden import tiny_prefill_case, tiny_projection_case
    p = tiny_prefill_case()
    res = oracle.mla_sparse_decode(p["q_nope"], p["q_pe"], p["kv_cache"], p["pe_cache"], p["end_pos"],
                                   p["topk_idx"], p["wkv_b"], p["scale"], cache_slot=p["cache_slot"])
    np.testing.assert_allclose(res.out.reshape(-1), np.array(g["prefill_out"]), rtol=1e-13, atol=1e-15)
    np.testing.assert_array_equal(np.isneginf(res.lse.reshape(-1)), np.isneginf(np.array(g["prefill_lse"])))
    fin = np.isfinite(res.lse.reshape(-1))
    np.testing.assert_allclose(res.lse.reshape(-1)[fin], np.array(g["prefill_lse"])[fin], rtol=1e-13)
    j = tiny_projection_case()
    np.testing.assert_allclose(oracle.output_projection(j["x"], j["wo"]).reshape(-1), np.array(g["projection"]),
                               rtol=1e-13, atol=1e-15)


def test_prefill_generator_structure():
    """One row per query position: slot = its sequence, end_pos = position
    + 1, and min(K, position + 1) distinct causally valid indices, -1 padded."""
    d = wl.generate_prefill(2, 40, 16, seed=7)
    R = 80
    pos = np.arange(R) % 40
    np.testing.assert_array_equal(d["cache_slot"].numpy(), np.arange(R) // 40)
    np.testing.assert_array_equal(d["end_pos"].numpy(), pos + 1)
    ti = d["topk_idx"].numpy()
    for r in range(R):
        n = min(16, pos[r] + 1)
        sel = ti[r, :n]
        assert len(set(sel.tolist())) == n and sel.min() >= 0 and sel.max() <= pos[r]
        assert np.all(ti[r, n:] == -1)
    assert tuple(d["kv_cache"].shape) == (2, 40, 512) and tuple(d["q_nope"].shape) == (R, 128, 128)
