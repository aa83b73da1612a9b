"""Python access to the fp64 CPU oracle (``mla_oracle.c``).

TEST INFRASTRUCTURE ONLY.  The oracle is the plain definition of the absorbed,
top-k masked MLA decode step (DeepSeek-V3.2-Exp atlas pages "Query-key
similarity", "Softmax" and "Apply value weights"; model.py 590-606).  Only the
tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this module.  It does not import the CUDA package, and the CUDA package
never imports it.

The C source is compiled with gcc into ``oracle/_build/liboracle.so`` on first
use (or by :func:`build`).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mla_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (fp64, OpenMP, IEEE semantics: no fast-math)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c99",
               "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        p = ctypes.c_void_p
        i = ctypes.c_int
        lib.oracle_mla_sparse_decode_f64.restype = ctypes.c_int
        lib.oracle_mla_sparse_decode_f64.argtypes = [
            p, p, p, p, p, i,            # q_nope q_pe kv pe wkv_b in_bf16
            p, p, ctypes.c_double,       # end_pos topk_idx scale
            i, i, i, i, i, i, i, i,      # B K S_max H Dn Dr Dl Dv
            p, i,                        # rows n_rows
            p, i,                        # cache_slot n_slots
            p, p, p, p, p,               # out lse q_lat o_lat w_full
        ]
        lib.oracle_output_projection_f64.restype = ctypes.c_int
        lib.oracle_output_projection_f64.argtypes = [p, p, i, i, i, i, p, i, p]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_num_threads.argtypes = []
        _lib = lib
    return _lib


def num_threads() -> int:
    """Threads the oracle's OpenMP loop uses (OMP_NUM_THREADS or all cores)."""
    return int(_load().oracle_num_threads())


def _dense(x, in_bf16: bool) -> np.ndarray:
    """Contiguous host array holding bf16 bit patterns (uint16) or float64."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if in_bf16:
                if x.dtype != torch.bfloat16:
                    raise TypeError("oracle: expected bfloat16 tensors")
                return x.view(torch.int16).numpy().view(np.uint16)
            return x.to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(x)
    if in_bf16:
        if a.dtype != np.uint16:
            raise TypeError("oracle: bf16 inputs must be uint16 bit patterns")
        return a
    return np.ascontiguousarray(a, dtype=np.float64)


def _ints(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x), dtype=np.int32)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


@dataclass
class OracleResult:
    out: np.ndarray                     # [n_rows, H, Dv]
    lse: np.ndarray                     # [n_rows, H]
    q_lat: np.ndarray | None = None     # [n_rows, H, Dl]
    o_lat: np.ndarray | None = None     # [n_rows, H, Dl]
    w_full: np.ndarray | None = None    # [n_rows, H, S_max]


def mla_sparse_decode(q_nope, q_pe, kv_cache, pe_cache, end_pos, topk_idx,
                      wkv_b, scale, rows=None, *, cache_slot=None, want_q_lat=False,
                      want_o_lat=False, want_weights=False) -> OracleResult:
    """Run the oracle on the given inputs.

    Shapes: q_nope [B,H,Dn], q_pe [B,H,Dr], kv_cache [B,S_max,Dl],
    pe_cache [B,S_max,Dr], end_pos [B], topk_idx [B,K],
    wkv_b [H*(Dn+Dv), Dl] or [H, Dn+Dv, Dl].  Dense inputs are all bfloat16
    (torch) / uint16 bit patterns (numpy), or all float64.  ``Dv`` is taken
    as ``Dn`` (the pages' qk_nope_head_dim = v_head_dim = 128) unless wkv_b is
    3-D, in which case Dv = wkv_b.shape[1] - Dn.

    ``rows`` selects batch rows (default: all); result r is batch row rows[r].
    ``cache_slot`` [B] (optional): row b reads kv_cache[cache_slot[b]] and
    pe_cache[cache_slot[b]] (the caches then hold n_slots = kv_cache.shape[0]
    sequences); the prefill of the page "Queries" is one row per query
    position with end_pos = position + 1.
    """
    import numbers
    try:
        import torch
        is_bf16 = isinstance(q_nope, torch.Tensor) and q_nope.dtype == torch.bfloat16
    except ImportError:  # pragma: no cover
        is_bf16 = False
    if not is_bf16 and isinstance(q_nope, np.ndarray) and q_nope.dtype == np.uint16:
        is_bf16 = True

    B, H, Dn = (int(s) for s in q_nope.shape)
    Dr = int(q_pe.shape[2])
    S_max, Dl = int(kv_cache.shape[1]), int(kv_cache.shape[2])
    K = int(topk_idx.shape[1])
    if len(wkv_b.shape) == 3:
        Dv = int(wkv_b.shape[1]) - Dn
    else:
        Dv = int(wkv_b.shape[0]) // H - Dn
    assert isinstance(scale, numbers.Real)

    qn = _dense(q_nope, is_bf16)
    qp = _dense(q_pe, is_bf16)
    kv = _dense(kv_cache, is_bf16)
    pe = _dense(pe_cache, is_bf16)
    wb = _dense(wkv_b, is_bf16)
    ep = _ints(end_pos)
    ti = _ints(topk_idx)
    rows_a = _ints(np.arange(B) if rows is None else rows).reshape(-1)
    n = int(rows_a.shape[0])
    slots = None if cache_slot is None else _ints(cache_slot).reshape(-1)
    n_slots = int(kv_cache.shape[0])
    if slots is not None:
        assert slots.shape[0] == B, "cache_slot must hold one slot per row"

    out = np.zeros((n, H, Dv), np.float64)
    lse = np.zeros((n, H), np.float64)
    ql = np.zeros((n, H, Dl), np.float64) if want_q_lat else None
    ol = np.zeros((n, H, Dl), np.float64) if want_o_lat else None
    wf = np.zeros((n, H, S_max), np.float64) if want_weights else None

    rc = _load().oracle_mla_sparse_decode_f64(
        _ptr(qn), _ptr(qp), _ptr(kv), _ptr(pe), _ptr(wb), int(is_bf16),
        _ptr(ep), _ptr(ti), float(scale),
        B, K, S_max, H, Dn, Dr, Dl, Dv,
        _ptr(rows_a), n, _ptr(slots), n_slots,
        _ptr(out), _ptr(lse), _ptr(ql), _ptr(ol), _ptr(wf))
    if rc != 0:
        raise RuntimeError(f"oracle failed with code {rc}")
    return OracleResult(out=out, lse=lse, q_lat=ql, o_lat=ol, w_full=wf)


def output_projection(x, wo, rows=None) -> np.ndarray:
    """delta[r, n] = sum_k x[rows[r], k] * wo[n, k] in float64 (the attention
    update of the atlas page "Attention update", model.py 607-608).

    ``x`` [B, n_in] (or [B, H, Dv], flattened per row) and ``wo`` [dim, n_in]:
    both bfloat16 (torch) / uint16 bit patterns (numpy), or both float64.
    Returns [len(rows), dim] (all rows by default).
    """
    try:
        import torch
        is_bf16 = isinstance(x, torch.Tensor) and x.dtype == torch.bfloat16
    except ImportError:  # pragma: no cover
        is_bf16 = False
    if not is_bf16 and isinstance(x, np.ndarray) and x.dtype == np.uint16:
        is_bf16 = True
    B = int(x.shape[0])
    n_in = 1
    for d in x.shape[1:]:
        n_in *= int(d)
    dim = int(wo.shape[0])
    assert int(np.prod(wo.shape[1:])) == n_in, "wo must be [dim, n_in]"
    xa = _dense(x, is_bf16).reshape(B, n_in)
    wa = _dense(wo, is_bf16).reshape(dim, n_in)
    rows_a = _ints(np.arange(B) if rows is None else rows).reshape(-1)
    out = np.zeros((int(rows_a.shape[0]), dim), np.float64)
    rc = _load().oracle_output_projection_f64(_ptr(xa), _ptr(wa), int(is_bf16), B, n_in, dim,
                                              _ptr(rows_a), int(rows_a.shape[0]), _ptr(out))
    if rc != 0:
        raise RuntimeError(f"oracle failed with code {rc}")
    return out
