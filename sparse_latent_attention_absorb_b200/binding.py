"""ctypes binding of ``libmla_sparse_decode.so`` (see include/mla_sparse_decode.h).

Argument marshalling only: these functions check shapes, dtypes and devices of
torch tensors, pass their device pointers and the current CUDA stream to the
C ABI, and raise on a non-zero status.  Every step of the decode runs in the
library's sm_100a kernels; there is no fallback path.  If the library has not
been built, loading it raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

from .build import LIB_PATH

H, D_NOPE, D_ROPE, D_LAT, D_V = 128, 128, 64, 512, 128
D_MODEL = 7168  # model width of the pages (wo: 128 * 128 -> 7168)

STATUS = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_WORKSPACE", 3: "MLA_ERR_CUDA",
          4: "MLA_ERR_DEVICE_TIMEOUT", 5: "MLA_ERR_BAD_INDEX", 6: "MLA_ERR_UNSUPPORTED"}

# Every symbol the public header declares.
EXPORTS = ("mla_status_string", "mla_num_splits", "mla_sparse_decode_workspace_size", "mla_sparse_decode",
           "mla_absorb_q", "mla_sparse_attend", "mla_combine_value_up", "mla_sparse_decode_noalloc",
           "mla_sparse_decode_host_workspace_size", "mla_sparse_decode_host", "mla_sparse_decode_host_input_layout",
           "mla_output_projection_workspace_size", "mla_output_projection",
           "mla_sparse_decode_project_workspace_size", "mla_sparse_decode_project", "mla_sparse_prefill",
           "mla_selftest_wait_timeout", "mla_check_topk_indices", "mla_set_index_checks",
           "mla_sparse_decode_heads_workspace_size", "mla_sparse_decode_heads",
           "mla_output_projection_shard_workspace_size", "mla_output_projection_shard", "mla_dequant_fp8_blocks",
           "mla_prepare_wo", "mla_output_projection_prepared")
STATIC_SCRATCH_BYTES = 32 << 20  # MLA_STATIC_SCRATCH_BYTES

_lib = None


class MLAError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, code)}")
        self.code = code


def load_library():
    """Load the CUDA library (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"CUDA library not built: {LIB_PATH} (run sparse_latent_attention_absorb_b200.build)")
    lib = ctypes.CDLL(LIB_PATH)
    p, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.mla_status_string.restype = ctypes.c_char_p
    lib.mla_status_string.argtypes = [i]
    lib.mla_num_splits.restype = i
    lib.mla_num_splits.argtypes = [i, i]
    lib.mla_sparse_decode_workspace_size.restype = sz
    lib.mla_sparse_decode_workspace_size.argtypes = [i, i, i]
    lib.mla_sparse_decode.restype = i
    lib.mla_sparse_decode.argtypes = [p, p, p, p, p, p, p, f, p, i, i, i, p, sz, p, p, p]
    lib.mla_absorb_q.restype = i
    lib.mla_absorb_q.argtypes = [p, p, p, i, p]
    lib.mla_sparse_attend.restype = i
    lib.mla_sparse_attend.argtypes = [p, p, p, p, p, p, f, p, p, i, i, i, i, p, p]
    lib.mla_combine_value_up.restype = i
    lib.mla_combine_value_up.argtypes = [p, p, p, p, p, i, i, p]
    lib.mla_sparse_decode_noalloc.restype = i
    lib.mla_sparse_decode_noalloc.argtypes = [p, p, p, p, p, p, p, f, p, i, i, i, p, p, p]
    lib.mla_sparse_decode_host_workspace_size.restype = sz
    lib.mla_sparse_decode_host_workspace_size.argtypes = [i, i, i]
    lib.mla_sparse_decode_host_input_layout.restype = sz
    lib.mla_sparse_decode_host_input_layout.argtypes = [i, i, i, p]
    lib.mla_sparse_decode_host.restype = i
    lib.mla_sparse_decode_host.argtypes = [p, p, p, p, p, p, p, f, p, i, i, i, p, sz, p, p, p]
    lib.mla_output_projection_workspace_size.restype = sz
    lib.mla_output_projection_workspace_size.argtypes = [i, i]
    lib.mla_output_projection.restype = i
    lib.mla_output_projection.argtypes = [p, p, p, i, i, p, sz, p, p]
    lib.mla_sparse_decode_project_workspace_size.restype = sz
    lib.mla_sparse_decode_project_workspace_size.argtypes = [i, i, i, i]
    lib.mla_sparse_decode_project.restype = i
    lib.mla_sparse_decode_project.argtypes = [p, p, p, p, p, p, p, f, p, p, i, i, i, i, p, sz, p, p, p]
    lib.mla_sparse_prefill.restype = i
    lib.mla_sparse_prefill.argtypes = [p, p, p, p, p, p, p, p, f, p, i, i, i, i, p, sz, p, p, p]
    lib.mla_check_topk_indices.restype = i
    lib.mla_check_topk_indices.argtypes = [p, p, i, i, i, p, p, p]
    lib.mla_set_index_checks.restype = i
    lib.mla_set_index_checks.argtypes = [i]
    lib.mla_sparse_decode_heads_workspace_size.restype = sz
    lib.mla_sparse_decode_heads_workspace_size.argtypes = [i, i, i, i]
    lib.mla_sparse_decode_heads.restype = i
    lib.mla_sparse_decode_heads.argtypes = [p, p, p, p, p, p, p, f, p, i, i, i, i, p, sz, p, p, p]
    lib.mla_output_projection_shard_workspace_size.restype = sz
    lib.mla_output_projection_shard_workspace_size.argtypes = [i, i, i]
    lib.mla_dequant_fp8_blocks.restype = i
    lib.mla_dequant_fp8_blocks.argtypes = [p, p, p, i, i, p]
    lib.mla_output_projection_shard.restype = i
    lib.mla_output_projection_shard.argtypes = [p, p, ctypes.c_longlong, p, i, i, i, p, sz, p, p]
    lib.mla_prepare_wo.restype = i
    lib.mla_prepare_wo.argtypes = [p, ctypes.c_longlong, i, i, p, p]
    lib.mla_output_projection_prepared.restype = i
    lib.mla_output_projection_prepared.argtypes = [p, p, p, i, i, i, p, sz, p, p]
    lib.mla_selftest_wait_timeout.restype = i
    lib.mla_selftest_wait_timeout.argtypes = [p, p, p]
    _lib = lib
    return lib


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _check(t: torch.Tensor, name: str, dtype, shape=None):
    # one cheap test on the hot path; the detailed checks below only run to
    # name what is wrong
    try:
        if t.is_cuda and t.dtype == dtype and (shape is None or t.shape == shape) and t.is_contiguous():
            return
    except AttributeError:
        pass
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")


def _raise(rc: int, where: str):
    if rc != 0:
        raise MLAError(rc, where)


_sizing_cache: dict = {}


def num_splits(B: int, K: int) -> int:
    """mla_num_splits for the current device (a pure function of the sizes and
    the device's SM count, so it is cached)."""
    key = ("splits", torch.cuda.current_device() if torch.cuda.is_available() else -1, B, K)
    v = _sizing_cache.get(key)
    if v is None:
        v = _sizing_cache[key] = int(load_library().mla_num_splits(B, K))
    return v


def workspace_size(B: int, K: int, S_max: int) -> int:
    """mla_sparse_decode_workspace_size for the current device (cached, as above)."""
    key = ("ws", torch.cuda.current_device() if torch.cuda.is_available() else -1, B, K, S_max)
    v = _sizing_cache.get(key)
    if v is None:
        v = _sizing_cache[key] = int(load_library().mla_sparse_decode_workspace_size(B, K, S_max))
    return v


def mla_sparse_decode(q_nope, q_pe, kv_cache, pe_cache, end_pos, topk_idx, wkv_b, scale, out=None, workspace=None,
                      lse_out=None, d_status=None, stream=None):
    """The whole decode step; returns ``out`` (bf16 [B,128,128])."""
    lib = load_library()
    B = q_nope.shape[0]
    S_max = kv_cache.shape[1]
    K = topk_idx.shape[1]
    bf = torch.bfloat16
    _check(q_nope, "q_nope", bf, (B, H, D_NOPE))
    _check(q_pe, "q_pe", bf, (B, H, D_ROPE))
    _check(kv_cache, "kv_cache", bf, (B, S_max, D_LAT))
    _check(pe_cache, "pe_cache", bf, (B, S_max, D_ROPE))
    _check(end_pos, "end_pos", torch.int32, (B,))
    _check(topk_idx, "topk_idx", torch.int32, (B, K))
    _check(wkv_b, "wkv_b", bf, (H * (D_NOPE + D_V), D_LAT))
    if out is None:
        out = torch.empty((B, H, D_V), dtype=bf, device=q_nope.device)
    _check(out, "out", bf, (B, H, D_V))
    if lse_out is not None:
        _check(lse_out, "lse_out", torch.float32, (B, H))
    if d_status is not None:
        _check(d_status, "d_status", torch.int32, (1,))
    need = workspace_size(B, K, S_max)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q_nope.device)
    _check(workspace, "workspace", torch.uint8)
    rc = lib.mla_sparse_decode(_ptr(q_nope), _ptr(q_pe), _ptr(kv_cache), _ptr(pe_cache), _ptr(end_pos),
                               _ptr(topk_idx), _ptr(wkv_b), float(scale), _ptr(out), B, K, S_max, _ptr(workspace),
                               workspace.numel(), _ptr(lse_out), _ptr(d_status), _stream(stream))
    _raise(rc, "mla_sparse_decode")
    return out


def mla_absorb_q(q_nope, wkv_b, q_lat=None, stream=None):
    lib = load_library()
    B = q_nope.shape[0]
    bf = torch.bfloat16
    _check(q_nope, "q_nope", bf, (B, H, D_NOPE))
    _check(wkv_b, "wkv_b", bf, (H * (D_NOPE + D_V), D_LAT))
    if q_lat is None:
        q_lat = torch.empty((B, H, D_LAT), dtype=bf, device=q_nope.device)
    _check(q_lat, "q_lat", bf, (B, H, D_LAT))
    _raise(lib.mla_absorb_q(_ptr(q_nope), _ptr(wkv_b), _ptr(q_lat), B, _stream(stream)), "mla_absorb_q")
    return q_lat


def _o_part_spec(B: int, n_split: int):
    """Shape and dtype of mla_sparse_attend's o_part for this split count."""
    if n_split == 1:
        return (B, H, D_LAT), torch.bfloat16
    return (B, n_split, H, D_LAT), torch.bfloat16


def mla_sparse_attend(q_lat, q_pe, kv_cache, pe_cache, end_pos, topk_idx, scale, o_part=None, lse_part=None,
                      d_status=None, stream=None):
    """Per-split outputs; returns (o_part, lse_part [B,S,128] f32).

    o_part is bf16 [B,S,128,512] (normalised mix per split) when S > 1, and the
    bf16 mixed latent [B,128,512] when each row is one split (S == 1)."""
    lib = load_library()
    B, S_max, K = q_lat.shape[0], kv_cache.shape[1], topk_idx.shape[1]
    n_split = num_splits(B, K)
    bf = torch.bfloat16
    _check(q_lat, "q_lat", bf, (B, H, D_LAT))
    _check(q_pe, "q_pe", bf, (B, H, D_ROPE))
    _check(kv_cache, "kv_cache", bf, (B, S_max, D_LAT))
    _check(pe_cache, "pe_cache", bf, (B, S_max, D_ROPE))
    _check(end_pos, "end_pos", torch.int32, (B,))
    _check(topk_idx, "topk_idx", torch.int32, (B, K))
    dev = q_lat.device
    o_shape, o_dtype = _o_part_spec(B, n_split)
    if o_part is None:
        o_part = torch.empty(o_shape, dtype=o_dtype, device=dev)
    if lse_part is None:
        lse_part = torch.empty((B, n_split, H), dtype=torch.float32, device=dev)
    _check(o_part, "o_part", o_dtype, o_shape)
    _check(lse_part, "lse_part", torch.float32, (B, n_split, H))
    rc = lib.mla_sparse_attend(_ptr(q_lat), _ptr(q_pe), _ptr(kv_cache), _ptr(pe_cache), _ptr(end_pos),
                               _ptr(topk_idx), float(scale), _ptr(o_part), _ptr(lse_part), B, K, S_max, n_split,
                               _ptr(d_status), _stream(stream))
    _raise(rc, "mla_sparse_attend")
    return o_part, lse_part


def mla_combine_value_up(o_part, lse_part, wkv_b, out=None, lse_out=None, stream=None):
    """Merge of the splits and W_UV; o_part / lse_part as mla_sparse_attend returns them."""
    lib = load_library()
    B, n_split = lse_part.shape[0], lse_part.shape[1]
    bf = torch.bfloat16
    o_shape, o_dtype = _o_part_spec(B, n_split)
    _check(o_part, "o_part", o_dtype, o_shape)
    _check(lse_part, "lse_part", torch.float32, (B, n_split, H))
    _check(wkv_b, "wkv_b", bf, (H * (D_NOPE + D_V), D_LAT))
    if out is None:
        out = torch.empty((B, H, D_V), dtype=bf, device=o_part.device)
    _check(out, "out", bf, (B, H, D_V))
    if lse_out is not None:
        _check(lse_out, "lse_out", torch.float32, (B, H))
    rc = lib.mla_combine_value_up(_ptr(o_part), _ptr(lse_part), _ptr(wkv_b), _ptr(out), _ptr(lse_out), B, n_split,
                                  _stream(stream))
    _raise(rc, "mla_combine_value_up")
    return out


def host_workspace_size(B: int, K: int, S_max: int) -> int:
    """mla_sparse_decode_host_workspace_size for the current device (cached)."""
    key = ("hws", torch.cuda.current_device() if torch.cuda.is_available() else -1, B, K, S_max)
    v = _sizing_cache.get(key)
    if v is None:
        v = _sizing_cache[key] = int(load_library().mla_sparse_decode_host_workspace_size(B, K, S_max))
    return v


def _check_host(t: torch.Tensor, name: str, dtype, shape):
    if (not isinstance(t, torch.Tensor) or t.is_cuda or t.dtype != dtype or t.shape != shape
            or not t.is_contiguous()):
        raise ValueError(f"{name}: expected a contiguous host tensor {dtype} {tuple(shape)}")


def mla_sparse_decode_host(q_nope, q_pe, end_pos, topk_idx, kv_cache, pe_cache, wkv_b, scale, out, workspace,
                           lse_out=None, d_status=None, stream=None):
    """The decode step with the per-call tensors in host memory (pin them for
    asynchronous copies): q_nope, q_pe, end_pos, topk_idx and out are CPU
    tensors; kv_cache, pe_cache, wkv_b and the workspace live on the device.
    Enqueued on `stream`; `out` is complete once the stream has passed it."""
    lib = load_library()
    B, K, S_max = q_nope.shape[0], topk_idx.shape[1], kv_cache.shape[1]
    bf = torch.bfloat16
    _check_host(q_nope, "q_nope", bf, (B, H, D_NOPE))
    _check_host(q_pe, "q_pe", bf, (B, H, D_ROPE))
    _check_host(end_pos, "end_pos", torch.int32, (B,))
    _check_host(topk_idx, "topk_idx", torch.int32, (B, K))
    _check_host(out, "out", bf, (B, H, D_V))
    _check(kv_cache, "kv_cache", bf, (B, S_max, D_LAT))
    _check(pe_cache, "pe_cache", bf, (B, S_max, D_ROPE))
    _check(wkv_b, "wkv_b", bf, (H * (D_NOPE + D_V), D_LAT))
    _check(workspace, "workspace", torch.uint8)
    rc = lib.mla_sparse_decode_host(q_nope.data_ptr(), q_pe.data_ptr(), end_pos.data_ptr(), topk_idx.data_ptr(),
                                    kv_cache.data_ptr(), pe_cache.data_ptr(), wkv_b.data_ptr(), float(scale),
                                    out.data_ptr(), B, K, S_max, workspace.data_ptr(), workspace.numel(),
                                    _ptr(lse_out), _ptr(d_status), _stream(stream))
    _raise(rc, "mla_sparse_decode_host")
    return out


def projection_workspace_size(B: int, dim: int) -> int:
    """mla_output_projection_workspace_size for the current device (cached)."""
    key = ("pws", torch.cuda.current_device() if torch.cuda.is_available() else -1, B, dim)
    v = _sizing_cache.get(key)
    if v is None:
        v = _sizing_cache[key] = int(load_library().mla_output_projection_workspace_size(B, dim))
    return v


def mla_output_projection(x, wo, delta=None, workspace=None, d_status=None, stream=None):
    """delta = x . wo^T (bf16 [B, dim]) for x bf16 [B,128,128] (or [B,16384])
    and wo bf16 [dim, 16384]."""
    lib = load_library()
    B = x.shape[0]
    dim = wo.shape[0]
    bf = torch.bfloat16
    if not (x.dim() == 2 and x.shape[1] == H * D_V):
        _check(x, "x", bf, (B, H, D_V))
    _check(x, "x", bf)
    _check(wo, "wo", bf, (dim, H * D_V))
    if delta is None:
        delta = torch.empty((B, dim), dtype=bf, device=x.device)
    _check(delta, "delta", bf, (B, dim))
    if d_status is not None:
        _check(d_status, "d_status", torch.int32, (1,))
    if workspace is None:
        need = projection_workspace_size(B, dim)
        if need == 0:
            raise MLAError(1, "mla_output_projection")
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    _check(workspace, "workspace", torch.uint8)
    rc = lib.mla_output_projection(_ptr(x), _ptr(wo), _ptr(delta), B, dim, _ptr(workspace), workspace.numel(),
                                   _ptr(d_status), _stream(stream))
    _raise(rc, "mla_output_projection")
    return delta


def project_workspace_size(B: int, K: int, S_max: int, dim: int) -> int:
    """mla_sparse_decode_project_workspace_size for the current device (cached)."""
    key = ("dpws", torch.cuda.current_device() if torch.cuda.is_available() else -1, B, K, S_max, dim)
    v = _sizing_cache.get(key)
    if v is None:
        v = _sizing_cache[key] = int(load_library().mla_sparse_decode_project_workspace_size(B, K, S_max, dim))
    return v


def mla_sparse_decode_project(q_nope, q_pe, kv_cache, pe_cache, end_pos, topk_idx, wkv_b, scale, wo, delta=None,
                              workspace=None, lse_out=None, d_status=None, stream=None):
    """The decode step followed by the output projection; returns delta
    (bf16 [B, dim], dim = wo.shape[0])."""
    lib = load_library()
    B, S_max, K = q_nope.shape[0], kv_cache.shape[1], topk_idx.shape[1]
    dim = wo.shape[0]
    bf = torch.bfloat16
    _check(q_nope, "q_nope", bf, (B, H, D_NOPE))
    _check(q_pe, "q_pe", bf, (B, H, D_ROPE))
    _check(kv_cache, "kv_cache", bf, (B, S_max, D_LAT))
    _check(pe_cache, "pe_cache", bf, (B, S_max, D_ROPE))
    _check(end_pos, "end_pos", torch.int32, (B,))
    _check(topk_idx, "topk_idx", torch.int32, (B, K))
    _check(wkv_b, "wkv_b", bf, (H * (D_NOPE + D_V), D_LAT))
    _check(wo, "wo", bf, (dim, H * D_V))
    if delta is None:
        delta = torch.empty((B, dim), dtype=bf, device=q_nope.device)
    _check(delta, "delta", bf, (B, dim))
    if lse_out is not None:
        _check(lse_out, "lse_out", torch.float32, (B, H))
    if d_status is not None:
        _check(d_status, "d_status", torch.int32, (1,))
    if workspace is None:
        need = project_workspace_size(B, K, S_max, dim)
        if need == 0:
            raise MLAError(1, "mla_sparse_decode_project")
        workspace = torch.empty(need, dtype=torch.uint8, device=q_nope.device)
    _check(workspace, "workspace", torch.uint8)
    rc = lib.mla_sparse_decode_project(_ptr(q_nope), _ptr(q_pe), _ptr(kv_cache), _ptr(pe_cache), _ptr(end_pos),
                                       _ptr(topk_idx), _ptr(wkv_b), float(scale), _ptr(wo), _ptr(delta), B, K,
                                       S_max, dim, _ptr(workspace), workspace.numel(), _ptr(lse_out),
                                       _ptr(d_status), _stream(stream))
    _raise(rc, "mla_sparse_decode_project")
    return delta


def mla_sparse_prefill(q_nope, q_pe, kv_cache, pe_cache, cache_slot, end_pos, topk_idx, wkv_b, scale, out=None,
                       workspace=None, lse_out=None, d_status=None, stream=None):
    """Sparse prefill: one row per query position; row r reads the latents of
    sequence cache_slot[r] (kv_cache [n_slots, S_max, 512]) up to its causal
    bound end_pos[r].  Returns ``out`` (bf16 [R,128,128])."""
    lib = load_library()
    R, K = q_nope.shape[0], topk_idx.shape[1]
    n_slots, S_max = kv_cache.shape[0], kv_cache.shape[1]
    bf = torch.bfloat16
    _check(q_nope, "q_nope", bf, (R, H, D_NOPE))
    _check(q_pe, "q_pe", bf, (R, H, D_ROPE))
    _check(kv_cache, "kv_cache", bf, (n_slots, S_max, D_LAT))
    _check(pe_cache, "pe_cache", bf, (n_slots, S_max, D_ROPE))
    _check(cache_slot, "cache_slot", torch.int32, (R,))
    _check(end_pos, "end_pos", torch.int32, (R,))
    _check(topk_idx, "topk_idx", torch.int32, (R, K))
    _check(wkv_b, "wkv_b", bf, (H * (D_NOPE + D_V), D_LAT))
    if out is None:
        out = torch.empty((R, H, D_V), dtype=bf, device=q_nope.device)
    _check(out, "out", bf, (R, H, D_V))
    if lse_out is not None:
        _check(lse_out, "lse_out", torch.float32, (R, H))
    if d_status is not None:
        _check(d_status, "d_status", torch.int32, (1,))
    if workspace is None:
        workspace = torch.empty(workspace_size(R, K, S_max), dtype=torch.uint8, device=q_nope.device)
    _check(workspace, "workspace", torch.uint8)
    rc = lib.mla_sparse_prefill(_ptr(q_nope), _ptr(q_pe), _ptr(kv_cache), _ptr(pe_cache), _ptr(cache_slot),
                                _ptr(end_pos), _ptr(topk_idx), _ptr(wkv_b), float(scale), _ptr(out), R, K, S_max,
                                n_slots, _ptr(workspace), workspace.numel(), _ptr(lse_out), _ptr(d_status),
                                _stream(stream))
    _raise(rc, "mla_sparse_prefill")
    return out


def selftest_wait_timeout(stream=None):
    """Runs the bounded-wait self-test (about 2 s); returns (status word,
    result bits) as the library wrote them: (MLA_ERR_DEVICE_TIMEOUT, 4) when
    healthy."""
    lib = load_library()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    result = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    _raise(lib.mla_selftest_wait_timeout(_ptr(status), _ptr(result), _stream(stream)), "mla_selftest_wait_timeout")
    torch.cuda.synchronize()
    return int(status.item()), int(result.item())


def mla_check_topk_indices(end_pos, topk_idx, S_max: int, d_status=None, row_flags=None, stream=None):
    """Repeated valid entries of the index rows (mla_check_topk_indices).
    Writes MLA_ERR_BAD_INDEX into d_status (int32 [1], if it holds 0) and 1/0
    per row into row_flags (int32 [B]); allocates row_flags when both are
    None.  Returns row_flags (or None)."""
    lib = load_library()
    B, K = topk_idx.shape
    _check(end_pos, "end_pos", torch.int32, (B,))
    _check(topk_idx, "topk_idx", torch.int32)
    if d_status is None and row_flags is None:
        row_flags = torch.empty(B, dtype=torch.int32, device=topk_idx.device)
    if row_flags is not None:
        _check(row_flags, "row_flags", torch.int32, (B,))
    if d_status is not None:
        _check(d_status, "d_status", torch.int32)
    rc = lib.mla_check_topk_indices(_ptr(end_pos), _ptr(topk_idx), B, K, S_max, _ptr(d_status), _ptr(row_flags),
                                    _stream(stream))
    _raise(rc, "mla_check_topk_indices")
    return row_flags


def set_index_checks(enable: bool) -> bool:
    """Turns the process-wide opt-in index validation on or off
    (mla_set_index_checks); returns the previous setting."""
    return bool(load_library().mla_set_index_checks(1 if enable else 0))


def mla_sparse_decode_heads(q_nope, q_pe, kv_cache, pe_cache, end_pos, topk_idx, wkv_b, scale, out=None,
                            workspace=None, lse_out=None, d_status=None, stream=None):
    """One tensor-parallel shard of the decode step: the heads of q_nope
    (bf16 [B, n_heads, 128]) with wkv_b holding their rows (bf16
    [n_heads*256, 512]); returns ``out`` (bf16 [B, n_heads, 128])."""
    lib = load_library()
    B, n_heads = q_nope.shape[0], q_nope.shape[1]
    S_max = kv_cache.shape[1]
    K = topk_idx.shape[1]
    bf = torch.bfloat16
    _check(q_nope, "q_nope", bf, (B, n_heads, D_NOPE))
    _check(q_pe, "q_pe", bf, (B, n_heads, D_ROPE))
    _check(kv_cache, "kv_cache", bf, (B, S_max, D_LAT))
    _check(pe_cache, "pe_cache", bf, (B, S_max, D_ROPE))
    _check(end_pos, "end_pos", torch.int32, (B,))
    _check(topk_idx, "topk_idx", torch.int32, (B, K))
    _check(wkv_b, "wkv_b", bf, (n_heads * (D_NOPE + D_V), D_LAT))
    if out is None:
        out = torch.empty((B, n_heads, D_V), dtype=bf, device=q_nope.device)
    _check(out, "out", bf, (B, n_heads, D_V))
    if lse_out is not None:
        _check(lse_out, "lse_out", torch.float32, (B, n_heads))
    if workspace is None:
        n = lib.mla_sparse_decode_heads_workspace_size(B, K, S_max, n_heads)
        if n == 0:
            raise MLAError(1, "mla_sparse_decode_heads_workspace_size")
        workspace = torch.empty(n, dtype=torch.uint8, device=q_nope.device)
    _check(workspace, "workspace", torch.uint8)
    rc = lib.mla_sparse_decode_heads(_ptr(q_nope), _ptr(q_pe), _ptr(kv_cache), _ptr(pe_cache), _ptr(end_pos),
                                     _ptr(topk_idx), _ptr(wkv_b), float(scale), _ptr(out), B, K, S_max, n_heads,
                                     _ptr(workspace), workspace.numel(), _ptr(lse_out), _ptr(d_status),
                                     _stream(stream))
    _raise(rc, "mla_sparse_decode_heads")
    return out


def mla_output_projection_shard(x, wo, delta=None, workspace=None, d_status=None, stream=None):
    """Row-parallel partial of the output projection: x bf16 [B, k_in] (a
    shard's flattened decode output), wo a bf16 [dim, k_in] view whose rows
    may be strided (a column slice of the full wo); returns delta bf16
    [B, dim] = x . wo^T."""
    lib = load_library()
    B, k_in = x.shape
    dim = wo.shape[0]
    _check(x, "x", torch.bfloat16, (B, k_in))
    if not (wo.is_cuda and wo.dtype == torch.bfloat16 and wo.dim() == 2 and wo.shape[1] == k_in and wo.stride(1) == 1):
        raise ValueError("wo: expected a CUDA bf16 [dim, k_in] view with unit column stride")
    if delta is None:
        delta = torch.empty((B, dim), dtype=torch.bfloat16, device=x.device)
    _check(delta, "delta", torch.bfloat16, (B, dim))
    if workspace is None:
        n = lib.mla_output_projection_shard_workspace_size(B, dim, k_in)
        if n == 0:
            raise MLAError(1, "mla_output_projection_shard_workspace_size")
        workspace = torch.empty(n, dtype=torch.uint8, device=x.device)
    _check(workspace, "workspace", torch.uint8)
    rc = lib.mla_output_projection_shard(_ptr(x), _ptr(wo), wo.stride(0), _ptr(delta), B, dim, k_in, _ptr(workspace),
                                         workspace.numel(), _ptr(d_status), _stream(stream))
    _raise(rc, "mla_output_projection_shard")
    return delta


class PreparedWo:
    """wo [dim, k_in] in the layout mla_output_projection_prepared streams
    (built once per weight by mla_prepare_wo): `data` is a bf16 device buffer
    of dim * k_in elements whose order is internal to the library."""

    def __init__(self, data, dim: int, k_in: int):
        self.data, self.dim, self.k_in = data, dim, k_in


def mla_prepare_wo(wo, stream=None) -> PreparedWo:
    """The prepared copy of wo, a bf16 [dim, k_in] CUDA view with unit column
    stride (its rows may be strided: a tensor-parallel column slice)."""
    lib = load_library()
    if not (wo.is_cuda and wo.dtype == torch.bfloat16 and wo.dim() == 2 and wo.stride(1) == 1):
        raise ValueError("wo: expected a CUDA bf16 [dim, k_in] view with unit column stride")
    dim, k_in = wo.shape
    data = torch.empty(dim * k_in, dtype=torch.bfloat16, device=wo.device)
    _raise(lib.mla_prepare_wo(_ptr(wo), wo.stride(0), dim, k_in, _ptr(data), _stream(stream)), "mla_prepare_wo")
    return PreparedWo(data, dim, k_in)


def mla_output_projection_prepared(x, wo_p: PreparedWo, delta=None, workspace=None, d_status=None, stream=None):
    """delta bf16 [B, dim] = x . wo^T from the prepared wo (bit-identical to
    mla_output_projection_shard on the original); x bf16 [B, k_in]."""
    lib = load_library()
    B, k_in = x.shape
    dim = wo_p.dim
    _check(x, "x", torch.bfloat16, (B, wo_p.k_in))
    if delta is None:
        delta = torch.empty((B, dim), dtype=torch.bfloat16, device=x.device)
    _check(delta, "delta", torch.bfloat16, (B, dim))
    if workspace is None:
        n = lib.mla_output_projection_shard_workspace_size(B, dim, k_in)
        if n == 0:
            raise MLAError(1, "mla_output_projection_shard_workspace_size")
        workspace = torch.empty(n, dtype=torch.uint8, device=x.device)
    _check(workspace, "workspace", torch.uint8)
    rc = lib.mla_output_projection_prepared(_ptr(x), _ptr(wo_p.data), _ptr(delta), B, dim, k_in, _ptr(workspace),
                                            workspace.numel(), _ptr(d_status), _stream(stream))
    _raise(rc, "mla_output_projection_prepared")
    return delta


def mla_dequant_fp8_blocks(w_fp8, scale, out=None, stream=None):
    """bf16 weight from E4M3 codes (uint8 [rows, cols], or a float8_e4m3fn
    tensor) and one f32 scale per 128 x 128 block; returns out (bf16
    [rows, cols])."""
    lib = load_library()
    if w_fp8.dtype != torch.uint8:
        w_fp8 = w_fp8.view(torch.uint8)
    rows, cols = w_fp8.shape
    _check(w_fp8, "w_fp8", torch.uint8, (rows, cols))
    _check(scale, "scale", torch.float32, ((rows + 127) // 128, (cols + 127) // 128))
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.bfloat16, device=w_fp8.device)
    _check(out, "out", torch.bfloat16, (rows, cols))
    _raise(lib.mla_dequant_fp8_blocks(_ptr(w_fp8), _ptr(scale), _ptr(out), rows, cols, _stream(stream)),
           "mla_dequant_fp8_blocks")
    return out


class Fp8Wkvb:
    """wkv_b held in fp8 with block scales, dequantised to bf16 on first use
    and kept (the decode excerpt's ``self.dequant_wkv_b``): ``weight()``
    returns the bf16 wkv_b that every decode entry point takes."""

    def __init__(self, w_fp8, scale):
        self.w_fp8, self.scale, self._bf16 = w_fp8, scale, None

    def weight(self, stream=None):
        if self._bf16 is None:
            self._bf16 = mla_dequant_fp8_blocks(self.w_fp8, self.scale, stream=stream)
        return self._bf16


def host_input_buffer(B: int, K: int, S_max: int):
    """A pinned host buffer laid out like the host entry point's staging area,
    and views of its four inputs (q_nope, q_pe, end_pos, topk_idx): filling
    the views and passing them to mla_sparse_decode_host uploads them in one
    copy."""
    lib = load_library()
    offs = (ctypes.c_size_t * 4)()
    total = lib.mla_sparse_decode_host_input_layout(B, K, S_max, offs)
    if total == 0:
        raise MLAError(1, "mla_sparse_decode_host_input_layout")
    buf = torch.empty(total, dtype=torch.uint8).pin_memory()

    def view(off, dtype, shape):
        n = 1
        for d_ in shape:
            n *= d_
        return buf[off:off + n * torch.tensor([], dtype=dtype).element_size()].view(dtype).view(shape)

    return buf, {"q_nope": view(offs[0], torch.bfloat16, (B, H, D_NOPE)),
                 "q_pe": view(offs[1], torch.bfloat16, (B, H, D_ROPE)),
                 "end_pos": view(offs[2], torch.int32, (B,)),
                 "topk_idx": view(offs[3], torch.int32, (B, K))}
