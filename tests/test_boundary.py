"""The C ABI on the host: the library loads and exports every declared symbol,
status strings, sizing functions and argument validation (which rejects bad
arguments before touching the GPU).  No kernel is launched here."""
import ctypes
import os
import re

import pytest

from sparse_latent_attention_absorb_b200 import binding, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "mla_sparse_decode.h")
INVALID_ARG, WORKSPACE = 1, 2


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return set(re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", text))


def test_header_declarations_match_binding_exports():
    assert declared_functions() == set(binding.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_exports_have_c_linkage():
    out = os.popen(f"nm -D --defined-only {build.LIB_PATH}").read()
    for name in declared_functions():
        assert re.search(rf"\bT {name}$", out, flags=re.M), name


def test_status_strings(lib):
    for code, name in binding.STATUS.items():
        assert lib.mla_status_string(code).decode() == name
    assert lib.mla_status_string(99).decode() == "MLA_ERR_UNKNOWN"


def test_num_splits_properties(lib):
    assert lib.mla_num_splits(0, 10) == 0 and lib.mla_num_splits(4, 0) == 0
    for B in (1, 2, 8, 16, 32, 64, 100, 1000):
        for K in (1, 31, 32, 33, 256, 2048, 8192):
            n = lib.mla_num_splits(B, K)
            assert 1 <= n <= max(1, -(-K // 32))
            assert n <= 128
            if B >= 74:
                assert n == 1


def test_workspace_size_formula(lib):
    for B, K in ((1, 256), (8, 2048), (64, 2048), (3, 100)):
        n = lib.mla_num_splits(B, K)
        got = lib.mla_sparse_decode_workspace_size(B, K, 4096)
        # q_lat bf16, per-split outputs (bf16; O~ itself with one split),
        # their log-sum-exps
        o_bytes = B * n * 128 * 512 * 2
        need = B * 128 * 512 * 2 + o_bytes + B * n * 128 * 4
        assert need <= got <= need + 3 * 256
    assert lib.mla_sparse_decode_workspace_size(0, 1, 1) == 0
    assert lib.mla_sparse_decode_workspace_size(1, 1, 0) == 0


def _fake(addr):
    return ctypes.c_void_p(addr)


def test_decode_rejects_bad_arguments_without_a_launch(lib):
    A = 0x10000  # aligned, never dereferenced: validation fails first
    good = [_fake(A)] * 7

    def call(ptrs=None, scale=0.07, B=2, K=16, S=32, out=_fake(A), ws=_fake(A), wsb=1 << 30, lse=None, st=None):
        p = ptrs or good
        return lib.mla_sparse_decode(*p[:6], p[6], ctypes.c_float(scale), out, B, K, S, ws, wsb, lse, st, None)

    for i in range(7):
        bad = list(good)
        bad[i] = None
        assert call(bad) == INVALID_ARG
        bad[i] = _fake(A + 8)  # misaligned
        assert call(bad) == INVALID_ARG
    assert call(out=None) == INVALID_ARG
    assert call(B=0) == INVALID_ARG
    assert call(K=0) == INVALID_ARG
    assert call(S=0) == INVALID_ARG
    assert call(scale=float("nan")) == INVALID_ARG
    assert call(scale=float("inf")) == INVALID_ARG
    assert call(lse=_fake(A + 2)) == INVALID_ARG
    assert call(st=_fake(A + 1)) == INVALID_ARG


def test_step_entry_points_reject_bad_arguments(lib):
    A = 0x10000
    assert lib.mla_absorb_q(None, _fake(A), _fake(A), 4, None) == INVALID_ARG
    assert lib.mla_absorb_q(_fake(A), _fake(A), _fake(A + 4), 4, None) == INVALID_ARG
    assert lib.mla_absorb_q(_fake(A), _fake(A), _fake(A), 0, None) == INVALID_ARG
    args = [_fake(A)] * 6
    assert lib.mla_sparse_attend(*args, ctypes.c_float(1.0), _fake(A), None, 2, 16, 32, 1, None, None) == INVALID_ARG
    assert lib.mla_sparse_attend(*args, ctypes.c_float(1.0), _fake(A), _fake(A), 2, 0, 32, 1, None, None) == INVALID_ARG
    assert lib.mla_combine_value_up(_fake(A), _fake(A), _fake(A), _fake(A), None, 2, 0, None) == INVALID_ARG
    assert lib.mla_combine_value_up(_fake(A), _fake(A), _fake(A), _fake(A), None, 2, 129, None) == INVALID_ARG
    assert lib.mla_combine_value_up(_fake(A), None, _fake(A), _fake(A), None, 2, 1, None) == INVALID_ARG


def test_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros((1, 128, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        binding.mla_absorb_q(x, torch.zeros((128 * 256, 512), dtype=torch.bfloat16))


def test_projection_workspace_size_formula(lib):
    sms = 148  # planning SM count without a visible GPU (B200)
    for B, dim in ((1, 7168), (64, 7168), (3, 128), (256, 1024), (300, 256)):
        y_tiles = -(-B // 256)
        n_tile = -(-(-(-B // y_tiles)) // 16) * 16
        tiles = y_tiles * (dim // 128)
        got = lib.mla_output_projection_workspace_size(B, dim)
        if tiles >= sms:
            assert got == 256  # one CTA per tile writes bf16 directly: no partials
        else:
            # units of four k-blocks for tiles of <= 64 rows, else of one; at
            # most one CTA per unit; two f32 partial slots per CTA
            units = tiles * (64 if n_tile <= 64 else 256)
            assert got == 2 * min(sms, units) * n_tile * 128 * 4
    assert lib.mla_output_projection_workspace_size(1000, 7168) == 256  # 4 x 56 tiles >= 148 SMs
    for B, dim in ((0, 7168), (1, 0), (1, 100), (1, 7169), (1, 1 << 17)):
        assert lib.mla_output_projection_workspace_size(B, dim) == 0
    # the fused call holds the decode scratch, the per-head outputs and the partials
    for B, K in ((64, 2048), (3, 100)):
        dec = lib.mla_sparse_decode_workspace_size(B, K, 4096)
        proj = lib.mla_output_projection_workspace_size(B, 7168)
        need = dec + B * 16384 * 2 + proj
        got = lib.mla_sparse_decode_project_workspace_size(B, K, 4096, 7168)
        assert need <= got <= need + 3 * 256
    assert lib.mla_sparse_decode_project_workspace_size(1, 1, 1, 100) == 0
    assert lib.mla_sparse_decode_project_workspace_size(0, 1, 1, 7168) == 0


def test_projection_rejects_bad_arguments_without_a_launch(lib):
    A = 0x10000
    ok = dict(x=_fake(A), wo=_fake(A), delta=_fake(A), B=4, dim=7168, ws=_fake(A), wsb=1 << 30, st=None)

    def call(**kw):
        a = dict(ok, **kw)
        return lib.mla_output_projection(a["x"], a["wo"], a["delta"], a["B"], a["dim"], a["ws"], a["wsb"], a["st"],
                                         None)

    for name in ("x", "wo", "delta"):
        assert call(**{name: None}) == INVALID_ARG
        assert call(**{name: _fake(A + 8)}) == INVALID_ARG
    for dim in (0, 64, 100, 7168 + 64, 1 << 17):
        assert call(dim=dim) == INVALID_ARG
    assert call(B=0) == INVALID_ARG
    assert call(st=_fake(A + 2)) == INVALID_ARG

    args = [_fake(A)] * 7
    base = dict(wo=_fake(A), delta=_fake(A), B=2, K=16, S=32, dim=7168, scale=0.07)

    def call_p(ptrs=None, **kw):
        a = dict(base, **kw)
        p = ptrs or args
        return lib.mla_sparse_decode_project(*p[:7], ctypes.c_float(a["scale"]), a["wo"], a["delta"], a["B"], a["K"],
                                             a["S"], a["dim"], _fake(A), 1 << 30, None, None, None)

    for i in range(7):
        bad = list(args)
        bad[i] = None
        assert call_p(bad) == INVALID_ARG
    assert call_p(wo=None) == INVALID_ARG
    assert call_p(delta=_fake(A + 4)) == INVALID_ARG
    assert call_p(dim=100) == INVALID_ARG
    assert call_p(K=0) == INVALID_ARG
    assert call_p(scale=float("nan")) == INVALID_ARG


def test_prefill_rejects_bad_arguments_without_a_launch(lib):
    A = 0x10000
    args = [_fake(A)] * 4

    def call(slot=_fake(A), n_slots=2, R=4, K=16, S=32, scale=0.07):
        return lib.mla_sparse_prefill(*args, slot, _fake(A), _fake(A), _fake(A), ctypes.c_float(scale), _fake(A), R,
                                      K, S, n_slots, _fake(A), 1 << 30, None, None, None)

    assert call(slot=None) == INVALID_ARG
    assert call(slot=_fake(A + 4)) == INVALID_ARG
    assert call(n_slots=0) == INVALID_ARG
    assert call(R=0) == INVALID_ARG
    assert call(K=0) == INVALID_ARG
    assert call(scale=float("inf")) == INVALID_ARG


def test_index_check_rejects_bad_arguments_without_a_launch(lib):
    A = 0x10000
    st = _fake(A)

    def call(ep=_fake(A), idx=_fake(A), B=2, K=16, S=32, status=st, flags=None):
        return lib.mla_check_topk_indices(ep, idx, B, K, S, status, flags, None)

    assert call(ep=None) == INVALID_ARG
    assert call(idx=None) == INVALID_ARG
    assert call(ep=_fake(A + 4)) == INVALID_ARG
    assert call(idx=_fake(A + 8)) == INVALID_ARG
    assert call(status=None, flags=None) == INVALID_ARG  # nothing to report into
    assert call(status=_fake(A + 2)) == INVALID_ARG
    assert call(status=None, flags=_fake(A + 1)) == INVALID_ARG
    assert call(B=0) == INVALID_ARG
    assert call(K=0) == INVALID_ARG
    assert call(S=0) == INVALID_ARG


def test_index_check_flag_is_a_process_wide_switch(lib):
    # a host-side flag only: nothing is launched
    prev = lib.mla_set_index_checks(1)
    try:
        assert lib.mla_set_index_checks(1) == 1
        assert lib.mla_set_index_checks(0) == 1
        assert lib.mla_set_index_checks(0) == 0
    finally:
        lib.mla_set_index_checks(prev)


def test_shard_entry_points_reject_bad_arguments_without_a_launch(lib):
    A = 0x10000
    p7 = [_fake(A)] * 7

    def dec(n_heads=64, B=2, K=16, S=32, ptrs=None, ws=_fake(A)):
        p = ptrs or p7
        return lib.mla_sparse_decode_heads(*p[:7], ctypes.c_float(0.07), _fake(A), B, K, S, n_heads, ws, 1 << 30,
                                           None, None, None)

    for n in (0, -1, 129):
        assert dec(n_heads=n) == INVALID_ARG
    for i in range(7):
        bad = list(p7)
        bad[i] = _fake(A + 4)
        assert dec(ptrs=bad) == INVALID_ARG
    assert lib.mla_sparse_decode_heads_workspace_size(2, 16, 32, 0) == 0
    assert lib.mla_sparse_decode_heads_workspace_size(2, 16, 32, 129) == 0
    # a shard's scratch scales with its heads; all 128 heads = the decode's
    assert lib.mla_sparse_decode_heads_workspace_size(64, 2048, 4096, 128) == \
        lib.mla_sparse_decode_workspace_size(64, 2048, 4096)
    assert lib.mla_sparse_decode_heads_workspace_size(64, 2048, 4096, 64) < \
        lib.mla_sparse_decode_workspace_size(64, 2048, 4096)

    def proj(k_in=8192, ld=16384, dim=7168, B=4, x=_fake(A), wo=_fake(A)):
        return lib.mla_output_projection_shard(x, wo, ld, _fake(A), B, dim, k_in, _fake(A), 1 << 30, None, None)

    for k_in in (0, 32, 100, 16384 + 64):
        assert proj(k_in=k_in) == INVALID_ARG
    for ld in (8191, 8196, 1 << 32):  # shorter than k_in, rows not 16-byte aligned, too long
        assert proj(ld=ld) == INVALID_ARG
    assert proj(dim=100) == INVALID_ARG
    assert proj(x=_fake(A + 8)) == INVALID_ARG
    assert lib.mla_output_projection_shard_workspace_size(4, 7168, 100) == 0
    assert lib.mla_output_projection_shard_workspace_size(4, 7168, 16384) == \
        lib.mla_output_projection_workspace_size(4, 7168)


def test_dequant_rejects_bad_arguments_without_a_launch(lib):
    A = 0x10000

    def call(w=_fake(A), s=_fake(A), o=_fake(A), rows=256, cols=512):
        return lib.mla_dequant_fp8_blocks(w, s, o, rows, cols, None)

    assert call(w=None) == INVALID_ARG
    assert call(o=_fake(A + 8)) == INVALID_ARG
    assert call(s=_fake(A + 2)) == INVALID_ARG
    assert call(rows=0) == INVALID_ARG
    assert call(cols=8) == INVALID_ARG
    assert call(cols=520 + 4) == INVALID_ARG


def test_prepared_projection_rejects_bad_arguments_without_a_launch(lib):
    A = 0x10000

    def prep(wo=_fake(A), ld=16384, dim=7168, k_in=16384, out=_fake(A)):
        return lib.mla_prepare_wo(wo, ld, dim, k_in, out, None)

    assert prep(wo=None) == INVALID_ARG
    assert prep(out=_fake(A + 8)) == INVALID_ARG
    for dim in (0, 64, 100, (1 << 16) + 128):
        assert prep(dim=dim) == INVALID_ARG
    for k_in in (0, 64, 192, 16384 + 256):  # whole 256-column blocks only
        assert prep(k_in=k_in) == INVALID_ARG
    for ld in (16383, 16380, 1 << 32):
        assert prep(ld=ld) == INVALID_ARG

    def proj(B=4, dim=7168, k_in=16384, x=_fake(A), w=_fake(A)):
        return lib.mla_output_projection_prepared(x, w, _fake(A), B, dim, k_in, _fake(A), 1 << 30, None, None)

    for k_in in (0, 64, 320, 16384 + 256):
        assert proj(k_in=k_in) == INVALID_ARG
    assert proj(B=0) == INVALID_ARG
    assert proj(dim=100) == INVALID_ARG
    assert proj(w=_fake(A + 4)) == INVALID_ARG
