"""Independent fp64 statements used to pin the oracle (tests only).

Each function computes the same result as the oracle by a different route
taken from the pages, so that a mistake in the oracle's arithmetic shows up as
a disagreement:

* ``nonabsorbed``: the "MHA prefill" form of the atlas page "Queries"
  (model.py 574-589): every cached latent is up-projected through wkv_b into
  per-head keys and values, the rotary key is appended, then the masked
  softmax mixes the values.  No absorption.
* ``transcript``: the decode excerpt of the page "Query-key similarity"
  (model.py 590-606) run as written in torch float64, with the indexer's
  output replaced by the given index row and the -inf/scatter mask built
  literally over all end_pos positions.

* ``prefill_transcript``: the "MHA prefill" excerpt of the page "Queries"
  (model.py 574-589) run as written in torch float64: every latent of the
  chunk up-projected through wkv_b, keys joined with the shared rotary key,
  the indexer's selection scattered into a -inf mask, the causal mask added.
* ``transcript_projection``: the output projection of the page "Attention
  update" (model.py 607-608), ``self.wo(x.flatten(2))``, as torch's
  ``F.linear`` in float64 on the [B, 1, H, Dv] head outputs.

None shares code with the oracle.
"""
from __future__ import annotations

import numpy as np
import torch


def to_f64(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        return x.detach().to(torch.float64).cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def valid_set(idx_row, ep: int) -> list[int]:
    return sorted({int(t) for t in np.asarray(idx_row).reshape(-1) if 0 <= int(t) < ep})


def nonabsorbed(q_nope, q_pe, kv, pe, wkv_b, end_pos, topk_idx, scale, Dv=None):
    """Per-row, per-head attention in up-projected (non-absorbed) form."""
    qn, qp, kv, pe, wb = (to_f64(a) for a in (q_nope, q_pe, kv, pe, wkv_b))
    B, H, Dn = qn.shape
    Dl = kv.shape[2]
    wb = wb.reshape(H, -1, Dl)
    if Dv is None:
        Dv = wb.shape[1] - Dn
    w_uk, w_uv = wb[:, :Dn, :], wb[:, Dn:Dn + Dv, :]
    out = np.zeros((B, H, Dv))
    for b in range(B):
        T = valid_set(np.asarray(topk_idx)[b], int(np.asarray(end_pos)[b]))
        if not T:
            continue
        c = kv[b, T, :]                                # [t, Dl]
        k_nope = np.einsum("hdc,tc->thd", w_uk, c)     # per-head keys
        v = np.einsum("hdc,tc->thd", w_uv, c)          # per-head values
        k_r = pe[b, T, :]                              # shared rotary key
        for h in range(H):
            q = np.concatenate([qn[b, h], qp[b, h]])
            k = np.concatenate([k_nope[:, h, :], k_r], axis=1)
            s = (k @ q) * scale
            a = np.exp(s - s.max())
            a /= a.sum()
            out[b, h] = a @ v[:, h, :]
    return out


def transcript(q_nope, q_pe, kv, pe, wkv_b, end_pos, topk_idx, scale, Dv=None):
    """The decode excerpt's einsums in torch float64, one batch row at a time
    (the excerpt uses one end_pos for the whole batch)."""
    qn, qp, kvt, pet, wb = (torch.as_tensor(to_f64(a)) for a in (q_nope, q_pe, kv, pe, wkv_b))
    B, H, Dn = qn.shape
    Dl = kvt.shape[2]
    wkv = wb.view(H, -1, Dl)
    if Dv is None:
        Dv = wkv.shape[1] - Dn
    outs = []
    for b in range(B):
        ep = int(np.asarray(end_pos)[b])
        T = valid_set(np.asarray(topk_idx)[b], ep)
        q_nope_b = qn[b:b + 1, None]                       # [1, 1, H, Dn]
        q_pe_b = qp[b:b + 1, None]
        q_abs = torch.einsum("bshd,hdc->bshc", q_nope_b, wkv[:, :Dn])
        scores = (torch.einsum("bshc,btc->bsht", q_abs, kvt[b:b + 1, :ep]) +
                  torch.einsum("bshr,btr->bsht", q_pe_b, pet[b:b + 1, :ep])) * scale
        topk_indices = torch.tensor([T], dtype=torch.int64).view(1, 1, -1)
        index_mask = torch.full((1, 1, ep), float("-inf"), dtype=torch.float64).scatter_(-1, topk_indices, 0)
        scores += index_mask.unsqueeze(2)
        scores = scores.softmax(dim=-1)
        x = torch.einsum("bsht,btc->bshc", scores, kvt[b:b + 1, :ep])
        x = torch.einsum("bshc,hdc->bshd", x, wkv[:, -Dv:])
        outs.append(x[0, 0])
    return torch.stack(outs).numpy()


def transcript_projection(x, wo):
    """``wo(x.flatten(2))`` of the page "Attention update": x holds the head
    outputs [B, H, Dv] of one position per row (or [B, H*Dv]); wo is the
    Linear weight [dim, H*Dv].  Returns [B, dim] in float64."""
    xt = torch.as_tensor(to_f64(x))
    B = xt.shape[0]
    x4 = xt.reshape(B, 1, -1, xt.shape[-1]) if xt.dim() == 3 else xt.reshape(B, 1, 1, -1)
    w = torch.as_tensor(to_f64(wo))
    return torch.nn.functional.linear(x4.flatten(2), w)[:, 0].numpy()


def prefill_transcript(q_nope, q_pe, kv, k_pe, wkv_b, topk_indices, scale, Dv):
    """q_nope [b,s,H,Dn], q_pe [b,s,H,Dr], kv [b,s,Dl] (the chunk's latents),
    k_pe [b,s,Dr], wkv_b [H*(Dn+Dv), Dl], topk_indices [b,s,K] (positions in
    [0, seqlen); ones after the query are removed by the causal mask).
    Returns x [b,s,H,Dv]."""
    qn, qp, kvt, kpe, wb = (torch.as_tensor(to_f64(a)) for a in (q_nope, q_pe, kv, k_pe, wkv_b))
    bsz, seqlen, n_heads, qk_nope = qn.shape
    q = torch.cat([qn, qp], dim=-1)
    kvu = torch.nn.functional.linear(kvt, wb)
    kvu = kvu.view(bsz, seqlen, n_heads, qk_nope + Dv)
    k_nope, v = torch.split(kvu, [qk_nope, Dv], dim=-1)
    k = torch.cat([k_nope, kpe.unsqueeze(2).expand(-1, -1, n_heads, -1)], dim=-1)
    scores = torch.einsum("bshd,bthd->bsht", q, k).mul_(scale)
    mask = torch.full((seqlen, seqlen), float("-inf"), dtype=torch.float64).triu_(1)
    idx = torch.as_tensor(np.asarray(topk_indices), dtype=torch.int64)
    index_mask = torch.full((bsz, seqlen, seqlen), float("-inf"), dtype=torch.float64).scatter_(-1, idx, 0)
    index_mask += mask
    scores += index_mask.unsqueeze(2)
    scores = scores.softmax(dim=-1)
    return torch.einsum("bsht,bthd->bshd", scores, v).numpy()
