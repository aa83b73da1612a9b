"""Seeded synthetic inputs for the sparse MLA decode step.

This module only draws random numbers and index sets; it holds none of the
attention arithmetic.  Both the CUDA path and the fp64 oracle are fed from it,
so the two always see identical bits.

Shapes follow DeepSeek-V3.2-Exp's decode step as the atlas pages show it
("Query-key similarity", decode excerpt model.py 590-606): 128 heads,
q_nope 128 wide, q_pe 64 wide, a 512-wide cached latent, a 64-wide cached
rotary key, and wkv_b viewed as [128 heads, 256, 512].

Distributions: q_nope, q_pe, kv_cache and pe_cache are bf16 draws of N(0,1);
wkv_b is bf16(N(0,1) * 512**-0.5); scale = fp32(192**-0.5).  For the output
projection that follows the step (wo: 16384 -> 7168, page "Attention update"),
its input x is a bf16 draw of N(0,1) and wo is bf16(N(0,1) * 16384**-0.5).  Every index row
holds distinct positions in [0, end_pos), shuffled (the indexer's top-k output
is in score order, not position order), padded with -1 up to K.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

H = 128          # heads
D_NOPE = 128     # qk_nope_head_dim
D_ROPE = 64      # qk_rope_head_dim
D_LAT = 512      # kv_lora_rank
D_V = 128        # v_head_dim
D_MODEL = 7168   # model width: wo maps H * D_V = 16384 -> 7168
SCALE = float(torch.tensor((D_NOPE + D_ROPE) ** -0.5, dtype=torch.float32))


@dataclass(frozen=True)
class Workload:
    """One synthetic decode workload.

    end_pos: (lo, hi) inclusive range of a uniform draw per row (lo == hi for a
    fixed length).  index: "uniform" | "recent" | "runs" | "dense".
    k_cap: the top-k budget; a row selects min(k_cap, end_pos) positions and
    the index tensor has K = k_cap columns (K = end_pos max for "dense").
    """
    name: str
    B: int
    S_max: int
    end_pos: tuple
    k_cap: int
    index: str
    seed: int
    recent: int = 0       # "recent": number of most recent positions taken
    run_len: int = 0      # "runs": length of each run
    n_runs: int = 0       # "runs": number of runs

    @property
    def K(self) -> int:
        return self.k_cap


# The pages' workloads (decode with 1001 cached positions on the pages; the
# longer contexts follow the DeepSeek-V3.2 top-2048 indexer budget).
WORKLOADS = {
    "b1_ctx1001_top256": Workload("b1_ctx1001_top256", 1, 1001, (1001, 1001), 256, "uniform", 1001),
    "b8_ctx4096_top2048": Workload("b8_ctx4096_top2048", 8, 4096, (4096, 4096), 2048, "uniform", 1002),
    "b32_ctx2k-8k_recent512_top2048": Workload(
        "b32_ctx2k-8k_recent512_top2048", 32, 8192, (2048, 8192), 2048, "recent", 1003, recent=512),
    "b64_ctx1k-32k_top2048": Workload("b64_ctx1k-32k_top2048", 64, 32768, (1024, 32768), 2048, "uniform", 1004),
    "b16_ctx131072_runs32x64": Workload(
        "b16_ctx131072_runs32x64", 16, 131072, (131072, 131072), 2048, "runs", 1005, run_len=64, n_runs=32),
    "b16_ctx8192_dense": Workload("b16_ctx8192_dense", 16, 8192, (8192, 8192), 8192, "dense", 1006),
}

# Reduced copies with the same index structure, small enough for the oracle
# to finish in seconds while still spanning several token tiles and a ragged
# tail.
SMALL_WORKLOADS = {
    "small_b2_ctx300_top100": Workload("small_b2_ctx300_top100", 2, 300, (300, 300), 100, "uniform", 2001),
    "small_b3_ctx1001_top256": Workload("small_b3_ctx1001_top256", 3, 1001, (1001, 1001), 256, "uniform", 2002),
    "small_b4_ctx600-2k_recent128_top400": Workload(
        "small_b4_ctx600-2k_recent128_top400", 4, 2048, (600, 2048), 400, "recent", 2003, recent=128),
    "small_b5_ctx40-700_top333": Workload("small_b5_ctx40-700_top333", 5, 704, (40, 700), 333, "uniform", 2004),
    "small_b2_ctx9000_runs6x37": Workload(
        "small_b2_ctx9000_runs6x37", 2, 9000, (9000, 9000), 222, "runs", 2005, run_len=37, n_runs=6),
    "small_b2_ctx500_dense": Workload("small_b2_ctx500_dense", 2, 500, (500, 500), 500, "dense", 2006),
    # enough rows that every row is one split of many tiles (online softmax
    # across tiles, the gather ring wrapping around, double-buffered P)
    "small_b80_ctx700_top300": Workload("small_b80_ctx700_top300", 80, 700, (700, 700), 300, "uniform", 2007),
    "small_b76_ctx150-2k_recent64_top700": Workload(
        "small_b76_ctx150-2k_recent64_top700", 76, 2048, (150, 2048), 700, "recent", 2008, recent=64),
    # few rows, so each row's index slots are split over many clusters: 32
    # and 18 key splits per row (the split merge reads them in batches of 16)
    "small_b1_ctx4096_top2048": Workload("small_b1_ctx4096_top2048", 1, 4096, (4096, 4096), 2048, "uniform", 2009),
    "small_b2_ctx1500-3k_top1100": Workload(
        "small_b2_ctx1500-3k_top1100", 2, 3000, (1500, 3000), 1100, "uniform", 2010),
}

ALL_WORKLOADS = {**WORKLOADS, **SMALL_WORKLOADS}


def _randperm(n: int, gen: torch.Generator) -> torch.Tensor:
    return torch.randperm(n, generator=gen, dtype=torch.int64)


def _runs(ep: int, run_len: int, n_runs: int, gen: torch.Generator) -> torch.Tensor:
    """n_runs non-overlapping runs of run_len consecutive positions, start
    offsets uniform in [0, ep - run_len] by rejection sampling."""
    assert n_runs * run_len <= ep
    starts: list[int] = []
    while len(starts) < n_runs:
        s = int(torch.randint(0, ep - run_len + 1, (1,), generator=gen))
        if all(s + run_len <= t or t + run_len <= s for t in starts):
            starts.append(s)
    return torch.cat([torch.arange(s, s + run_len) for s in starts])


def make_indices(w: Workload, gen: torch.Generator):
    """end_pos [B] int32 and topk_idx [B, K] int32 (-1 padded, shuffled)."""
    lo, hi = w.end_pos
    if lo == hi:
        end_pos = torch.full((w.B,), lo, dtype=torch.int64)
    else:
        end_pos = torch.randint(lo, hi + 1, (w.B,), generator=gen)
    K = w.K
    idx = torch.full((w.B, K), -1, dtype=torch.int64)
    for b in range(w.B):
        ep = int(end_pos[b])
        k = min(w.k_cap, ep)
        if w.index == "uniform":
            sel = _randperm(ep, gen)[:k]
        elif w.index == "dense":
            sel = _randperm(ep, gen)
        elif w.index == "recent":
            # all `recent` most recent positions, the rest distinct uniform
            # draws from the older part of the cache
            r = min(w.recent, k)
            recent = torch.arange(ep - r, ep)
            older = _randperm(ep - r, gen)[: k - r]
            sel = torch.cat([recent, older])
        elif w.index == "runs":
            sel = _runs(ep, w.run_len, w.n_runs, gen)[:k]
        else:
            raise ValueError(w.index)
        sel = sel[_randperm(sel.numel(), gen)]
        idx[b, : sel.numel()] = sel
    return end_pos.to(torch.int32), idx.to(torch.int32)


def _bf16_normal(shape, gen: torch.Generator, std: float = 1.0, chunk_dim0: bool = False):
    if not chunk_dim0:
        x = torch.randn(shape, generator=gen, dtype=torch.float32)
        if std != 1.0:
            x = x * std
        return x.to(torch.bfloat16)
    out = torch.empty(shape, dtype=torch.bfloat16)
    for i in range(shape[0]):
        x = torch.randn(shape[1:], generator=gen, dtype=torch.float32)
        if std != 1.0:
            x = x * std
        out[i] = x.to(torch.bfloat16)
    return out


def generate(w: Workload | str, seed_offset: int = 0, caches: bool = True) -> dict:
    """All inputs of one decode call, on the CPU.

    Returns a dict with q_nope [B,128,128], q_pe [B,128,64],
    kv_cache [B,S_max,512], pe_cache [B,S_max,64] (bf16), end_pos [B] and
    topk_idx [B,K] (int32), wkv_b [128*256, 512] (bf16), scale (float) and the
    workload.  ``seed_offset`` draws an independent set of the same shape;
    ``caches=False`` skips the (large) caches.
    """
    if isinstance(w, str):
        w = ALL_WORKLOADS[w]
    gen = torch.Generator().manual_seed(w.seed + 7919 * seed_offset)
    end_pos, topk_idx = make_indices(w, gen)
    d = {
        "workload": w,
        "end_pos": end_pos,
        "topk_idx": topk_idx,
        "q_nope": _bf16_normal((w.B, H, D_NOPE), gen),
        "q_pe": _bf16_normal((w.B, H, D_ROPE), gen),
        "wkv_b": _bf16_normal((H * (D_NOPE + D_V), D_LAT), gen, std=D_LAT ** -0.5),
        "scale": SCALE,
    }
    if caches:
        big = w.B * w.S_max * D_LAT > (1 << 26)
        d["kv_cache"] = _bf16_normal((w.B, w.S_max, D_LAT), gen, chunk_dim0=big)
        d["pe_cache"] = _bf16_normal((w.B, w.S_max, D_ROPE), gen, chunk_dim0=big)
    return d


def selected_count(end_pos: torch.Tensor, topk_idx: torch.Tensor) -> int:
    """Total number of valid (row, index) entries: sum over rows of |T_b|
    for distinct inputs."""
    ep = end_pos.to(torch.int64).unsqueeze(1)
    t = topk_idx.to(torch.int64)
    return int(((t >= 0) & (t < ep)).sum())


def generate_projection(B: int, dim: int = D_MODEL, seed: int = 2001) -> dict:
    """Inputs of one output projection, on the CPU: x bf16 [B, 16384] (the
    flattened per-head outputs of B rows) and wo bf16 [dim, 16384]."""
    gen = torch.Generator().manual_seed(seed)
    n_in = H * D_V
    return {
        "x": _bf16_normal((B, n_in), gen),
        "wo": _bf16_normal((dim, n_in), gen, std=n_in ** -0.5, chunk_dim0=dim * n_in > (1 << 26)),
    }


def generate_prefill(B: int, seqlen: int, K: int, seed: int = 2101) -> dict:
    """Inputs of one sparse prefill (page "Queries", prefill mode), on the CPU,
    one row per query position: q_nope [B*seqlen,128,128], q_pe
    [B*seqlen,128,64], kv_cache [B,seqlen,512], pe_cache [B,seqlen,64] (bf16;
    the chunk's own latents), cache_slot, end_pos and topk_idx [B*seqlen, K]
    (int32), wkv_b and scale.  Row b*seqlen + s is the query at position s of
    sequence b: end_pos = s + 1 (causal), and its index row holds
    min(K, s + 1) distinct positions of [0, s] in shuffled order (all of them
    while s < K, as an indexer whose scores are causally masked returns),
    -1 padded."""
    gen = torch.Generator().manual_seed(seed)
    R = B * seqlen
    pos = torch.arange(R, dtype=torch.int64) % seqlen
    topk = torch.full((R, K), -1, dtype=torch.int32)
    for r in range(R):
        s = int(pos[r])
        n = min(K, s + 1)
        sel = torch.randperm(s + 1, generator=gen)[:n]
        topk[r, :n] = sel.to(torch.int32)
    return {
        "q_nope": _bf16_normal((R, H, D_NOPE), gen),
        "q_pe": _bf16_normal((R, H, D_ROPE), gen),
        "kv_cache": _bf16_normal((B, seqlen, D_LAT), gen),
        "pe_cache": _bf16_normal((B, seqlen, D_ROPE), gen),
        "cache_slot": (torch.arange(R, dtype=torch.int64) // seqlen).to(torch.int32),
        "end_pos": (pos + 1).to(torch.int32),
        "topk_idx": topk,
        "wkv_b": _bf16_normal((H * (D_NOPE + D_V), D_LAT), gen, std=D_LAT ** -0.5),
        "scale": SCALE,
        "B": B, "seqlen": seqlen,
    }


def generate_fp8_wkv_b(n_heads: int = H, seed: int = 2201) -> dict:
    """wkv_b in the fp8 block format the decode excerpt can find it in
    (``wkv_b.weight`` with ``wkv_b.scale``), on the CPU: codes uint8
    [n_heads*256, 512] (OCP E4M3) and scale f32 [n_heads*2, 4], one per
    128 x 128 block.  Drawn as bf16-distributed weights N(0, 512^-0.5), each
    block scaled so that its largest magnitude maps to 448 (the largest E4M3
    value) and converted by torch's float8_e4m3fn cast."""
    gen = torch.Generator().manual_seed(seed)
    rows, cols = n_heads * (D_NOPE + D_V), D_LAT
    w = torch.randn((rows, cols), generator=gen, dtype=torch.float32) * D_LAT ** -0.5
    blocks = w.view(rows // 128, 128, cols // 128, 128)
    amax = blocks.abs().amax(dim=(1, 3)).clamp_min(1e-12)
    scale = (amax / 448.0).to(torch.float32)
    q = (blocks / scale[:, None, :, None]).view(rows, cols)
    codes = q.to(torch.float8_e4m3fn).view(torch.uint8)
    return {"codes": codes.contiguous(), "scale": scale.contiguous()}
