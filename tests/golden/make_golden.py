"""Writes oracle_tiny_regression.json from the fp64 oracle alone.

Run from the repository root:  python -m tests.golden.make_golden
The stored values come from ``oracle.mla_sparse_decode`` on ``tiny_case()``
and nothing else.
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


if __name__ == "__main__":
    main()
