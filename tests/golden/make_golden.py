"""Writes oracle_tiny_regression.json and oracle_next_rows_regression.json
from the fp64 oracle alone.

Run from the repository root:  python -m tests.golden.make_golden
The stored values come from ``oracle.mla_sparse_decode`` on ``tiny_case()``,
from the same call with per-row cache slots on ``tiny_prefill_case()`` and
from ``oracle.output_projection`` on ``tiny_projection_case()``, and nothing
else.
"""
import json
import os

import numpy as np


def tiny_case():
    """Seeded fp64 case: B=2, H=3, Dn=4, Dr=2, Dl=5, Dv=3, S_max=11, K=6."""
    rng = np.random.default_rng(20261202)
    B, H, Dn, Dr, Dl, Dv, S, K = 2, 3, 4, 2, 5, 3, 11, 6
    idx = np.full((B, K), -1, np.int32)
    idx[0, :5] = [9, 2, 4, 0, 7]
    idx[1, :6] = [3, 8, 1, 5, 6, 2]
    return dict(q_nope=rng.standard_normal((B, H, Dn)), q_pe=rng.standard_normal((B, H, Dr)),
                kv_cache=rng.standard_normal((B, S, Dl)), pe_cache=rng.standard_normal((B, S, Dr)),
                wkv_b=rng.standard_normal((H * (Dn + Dv), Dl)) / np.sqrt(Dl),
                end_pos=np.array([10, 9], np.int32), topk_idx=idx, scale=(Dn + Dr) ** -0.5)


def tiny_prefill_case():
    """tiny_case()'s two caches as two sequences; five query rows with their
    own slots, causal end positions and index rows (one later position in
    row 1, removed by its causal bound; row 4's slot does not exist)."""
    c = tiny_case()
    rng = np.random.default_rng(20261203)
    R, H, Dn, Dr = 5, 3, 4, 2
    c["q_nope"] = rng.standard_normal((R, H, Dn))
    c["q_pe"] = rng.standard_normal((R, H, Dr))
    c["cache_slot"] = np.array([0, 0, 1, 1, 2], np.int32)
    c["end_pos"] = np.array([3, 6, 1, 11, 4], np.int32)
    idx = np.full((R, 6), -1, np.int32)
    idx[0, :3] = [2, 0, 1]
    idx[1, :4] = [5, 9, 3, 0]
    idx[2, :1] = [0]
    idx[3, :6] = [10, 4, 7, 1, 8, 2]
    idx[4, :2] = [1, 3]
    c["topk_idx"] = idx
    return c


def tiny_projection_case():
    """Seeded fp64 case: B=3 rows of 2 heads x 3 values (n_in = 6), dim = 4."""
    rng = np.random.default_rng(20261204)
    return dict(x=rng.standard_normal((3, 2, 3)), wo=rng.standard_normal((4, 6)) / np.sqrt(6))


def main():
    import oracle
    c = tiny_case()
    res = oracle.mla_sparse_decode(c["q_nope"], c["q_pe"], c["kv_cache"], c["pe_cache"], c["end_pos"],
                                   c["topk_idx"], c["wkv_b"], c["scale"])
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny_regression.json")
    with open(path, "w") as f:
        json.dump({"_source": "written by tests/golden/make_golden.py from the fp64 oracle only",
                   "out": [float(x) for x in res.out.reshape(-1)],
                   "lse": [float(x) for x in res.lse.reshape(-1)]}, f, indent=1)
        f.write("\n")
    p = tiny_prefill_case()
    pres = oracle.mla_sparse_decode(p["q_nope"], p["q_pe"], p["kv_cache"], p["pe_cache"], p["end_pos"],
                                    p["topk_idx"], p["wkv_b"], p["scale"], cache_slot=p["cache_slot"])
    j = tiny_projection_case()
    delta = oracle.output_projection(j["x"], j["wo"])
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_next_rows_regression.json")
    with open(path, "w") as f:
        json.dump({"_source": "written by tests/golden/make_golden.py from the fp64 oracle only",
                   "prefill_out": [float(x) for x in pres.out.reshape(-1)],
                   "prefill_lse": [float(x) for x in pres.lse.reshape(-1)],
                   "projection": [float(x) for x in delta.reshape(-1)]}, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()
