"""The host-buffer entry point, mla_sparse_decode_host: per-call inputs and
output in (pinned) host memory, caches and weights on the device.  It must
give, bit for bit, what mla_sparse_decode gives on the same inputs, also when
consecutive calls alternate between two streams with their own workspaces."""
import ctypes

import pytest
import torch

import sparse_latent_attention_absorb_b200 as pkg
from sparse_latent_attention_absorb_b200 import binding
from sparse_latent_attention_absorb_b200 import workloads as wl

DEV = torch.device("cuda:0")
INVALID_ARG, WORKSPACE = 1, 2


def test_host_workspace_covers_decode_scratch_and_staging():
    lib = binding.load_library()
    for B, K, S in ((1, 256, 1001), (64, 2048, 32768), (7, 100, 300)):
        ws = lib.mla_sparse_decode_workspace_size(B, K, S)
        staged = B * 128 * 128 * 2 + B * 128 * 64 * 2 + B * 4 + B * K * 4 + B * 128 * 128 * 2
        got = lib.mla_sparse_decode_host_workspace_size(B, K, S)
        assert ws + staged <= got <= ws + staged + 5 * 256
    assert lib.mla_sparse_decode_host_workspace_size(0, 1, 1) == 0


def test_host_entry_rejects_bad_arguments_without_a_launch():
    lib = binding.load_library()
    A = ctypes.c_void_p(0x10000)
    args = [A] * 7
    assert lib.mla_sparse_decode_host(None, *args[1:], ctypes.c_float(0.07), A, 2, 16, 32, A, 1 << 30, None, None,
                                      None) == INVALID_ARG
    assert lib.mla_sparse_decode_host(*args, ctypes.c_float(0.07), A, 2, 0, 32, A, 1 << 30, None, None,
                                      None) == INVALID_ARG


def _pinned(t):
    return t.contiguous().pin_memory()


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["small_b80_ctx700_top300", "small_b4_ctx600-2k_recent128_top400"])
def test_host_entry_matches_device_entry(name):
    d = wl.generate(name)
    B, K, S = d["q_nope"].shape[0], d["topk_idx"].shape[1], d["kv_cache"].shape[1]
    kv, pe, w = d["kv_cache"].to(DEV), d["pe_cache"].to(DEV), d["wkv_b"].to(DEV)
    ref = pkg.mla_sparse_decode(d["q_nope"].to(DEV), d["q_pe"].to(DEV), kv, pe, d["end_pos"].to(DEV),
                                d["topk_idx"].to(DEV), w, d["scale"])
    hin = {k: _pinned(d[k]) for k in ("q_nope", "q_pe", "end_pos", "topk_idx")}
    out = torch.empty((B, 128, 128), dtype=torch.bfloat16).pin_memory()
    ws = torch.empty(pkg.host_workspace_size(B, K, S), dtype=torch.uint8, device=DEV)
    pkg.mla_sparse_decode_host(hin["q_nope"], hin["q_pe"], hin["end_pos"], hin["topk_idx"], kv, pe, w, d["scale"],
                               out, ws)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.cpu().view(torch.int16))


@pytest.mark.gpu
def test_host_entry_on_two_alternating_streams():
    name = "small_b5_ctx40-700_top333"
    base = wl.generate(name)
    sets = [base] + [wl.generate(name, seed_offset=i, caches=False) for i in (1, 2, 3)]
    B, K, S = base["q_nope"].shape[0], base["topk_idx"].shape[1], base["kv_cache"].shape[1]
    kv, pe = base["kv_cache"].to(DEV), base["pe_cache"].to(DEV)
    ws = [torch.empty(pkg.host_workspace_size(B, K, S), dtype=torch.uint8, device=DEV) for _ in range(2)]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [torch.empty((B, 128, 128), dtype=torch.bfloat16).pin_memory() for _ in sets]
    ws_w = [s_["wkv_b"].to(DEV) for s_ in sets]
    hins = [{k: _pinned(s_[k]) for k in ("q_nope", "q_pe", "end_pos", "topk_idx")} for s_ in sets]
    torch.cuda.synchronize()
    for i, s_ in enumerate(sets):
        h = hins[i]
        pkg.mla_sparse_decode_host(h["q_nope"], h["q_pe"], h["end_pos"], h["topk_idx"], kv, pe, ws_w[i],
                                   s_["scale"], outs[i], ws[i % 2], stream=streams[i % 2])
    torch.cuda.synchronize()
    for i, s_ in enumerate(sets):
        ref = pkg.mla_sparse_decode(s_["q_nope"].to(DEV), s_["q_pe"].to(DEV), kv, pe, s_["end_pos"].to(DEV),
                                    s_["topk_idx"].to(DEV), ws_w[i], s_["scale"])
        assert torch.equal(outs[i].view(torch.int16), ref.cpu().view(torch.int16))


def test_packed_input_layout_matches_the_staging_offsets():
    lib = binding.load_library()
    for B, K, S in ((1, 256, 1001), (64, 2048, 32768), (7, 100, 300)):
        offs = (ctypes.c_size_t * 4)()
        total = lib.mla_sparse_decode_host_input_layout(B, K, S, offs)
        sizes = [B * 128 * 128 * 2, B * 128 * 64 * 2, B * 4, B * K * 4]
        assert offs[0] == 0
        for i in range(3):  # each tensor follows the previous one, 256-byte aligned
            assert offs[i + 1] == -(-(offs[i] + sizes[i]) // 256) * 256
        assert total == offs[3] + sizes[3]
    assert lib.mla_sparse_decode_host_input_layout(0, 1, 1, None) == 0


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["small_b80_ctx700_top300", "small_b2_ctx300_top100"])
def test_packed_host_inputs_match_separate_ones(name):
    d = wl.generate(name)
    B, K, S = d["q_nope"].shape[0], d["topk_idx"].shape[1], d["kv_cache"].shape[1]
    kv, pe, w = d["kv_cache"].to(DEV), d["pe_cache"].to(DEV), d["wkv_b"].to(DEV)
    buf, views = binding.host_input_buffer(B, K, S)
    for k, v in views.items():
        v.copy_(d[k])
    ws = torch.empty(pkg.host_workspace_size(B, K, S), dtype=torch.uint8, device=DEV)
    out_packed = torch.empty((B, 128, 128), dtype=torch.bfloat16).pin_memory()
    pkg.mla_sparse_decode_host(views["q_nope"], views["q_pe"], views["end_pos"], views["topk_idx"], kv, pe, w,
                               d["scale"], out_packed, ws)
    torch.cuda.synchronize()
    hin = {k: _pinned(d[k]) for k in ("q_nope", "q_pe", "end_pos", "topk_idx")}
    out_sep = torch.empty((B, 128, 128), dtype=torch.bfloat16).pin_memory()
    pkg.mla_sparse_decode_host(hin["q_nope"], hin["q_pe"], hin["end_pos"], hin["topk_idx"], kv, pe, w, d["scale"],
                               out_sep, ws)
    torch.cuda.synchronize()
    assert torch.equal(out_packed.view(torch.int16), out_sep.view(torch.int16))
