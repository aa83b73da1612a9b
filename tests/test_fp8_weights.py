"""fp8 wkv_b (page "Query-key similarity", decode excerpt, model.py 591-592:
``self.dequant_wkv_b = weight_dequant(self.wkv_b.weight, self.wkv_b.scale)``,
built once and used in place of wkv_b).  The pages do not print the block
format; the reading (DeepSeek-V3's): E4M3 codes, one f32 scale per 128 x 128
block, w = bf16(e4m3 * scale) with the product exact and rounded once.

CPU: the oracle (``oracle/dequant.py``) pinned to the E4M3 definition through
torch's float8_e4m3fn cast, to hand-derived values (including a tie and a
product whose double rounding through float32 would differ), and to exact
rational arithmetic on random samples.
GPU: the kernel bit-exact against the oracle at the full size of wkv_b, and the
decode with the dequantised weight against the fp64 decode.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import dequant as dq
from sparse_latent_attention_absorb_b200 import workloads as wl

ALL_CODES = np.arange(256, dtype=np.uint8)


def test_e4m3_values_match_torch_float8_cast():
    ours = dq.e4m3_value(ALL_CODES)
    ref = torch.from_numpy(ALL_CODES).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    assert np.isnan(ours).sum() == 2  # 0x7F, 0xFF
    assert np.nanmax(ours) == 448.0 and np.nanmin(np.abs(ours[ours != 0])) == 2.0 ** -9


# (code, scale bits, expected bf16 bits), each derived by hand:
HAND = [
    (0x38, 0x3F000000, 0x3F00),  # 1.0 * 0.5 = 0.5
    (0xB8, 0x3F000000, 0xBF00),  # -1.0 * 0.5 = -0.5
    (0x01, 0x40400000, 0x3BC0),  # subnormal 2^-9 * 3 = 1.5 * 2^-8
    (0x7E, 0x3F802000, 0x43E0),  # 448 * (1 + 2^-10) = 448.4375 -> 448 (bf16 step 2 there)
    (0x38, 0x3F808000, 0x3F80),  # 1 * (1 + 2^-8): halfway between 1 and 1 + 2^-7 -> even: 1
    (0x38, 0x3F818000, 0x3F82),  # 1 * (1 + 3 * 2^-8): halfway -> even: 1 + 2^-6
    # -384 * 0x3F99AAAB = -(461 + 2^-16): just past the 460/462 midpoint -> -462;
    # through float32 first it would become the tie -461 and then -460 (0xC3E6)
    (0xFC, 0x3F99AAAB, 0xC3E7),
]


def _scale_value(bits):
    return float(np.array([bits], dtype=np.uint32).view(np.float32)[0])


@pytest.mark.parametrize("code,sbits,want", HAND)
def test_hand_derived_dequant_values(code, sbits, want):
    got = dq.dequant(np.full((128, 128), code, np.uint8), np.array([[_scale_value(sbits)]], np.float32))
    assert np.all(got == want)


def test_unit_and_power_of_two_scales_are_exact():
    codes = ALL_CODES[(ALL_CODES & 0x7F) != 0x7F]
    vals = dq.e4m3_value(codes)
    for k in (-20, -3, 0, 5):
        got = dq.bf16_round(vals * 2.0 ** k)
        want = torch.from_numpy(vals * 2.0 ** k).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(got, want)  # exact values: no rounding happens


def _nearest_bf16_exact(x: Fraction) -> int:
    """Nearest bf16 to a rational by enumeration of the neighbouring bit
    patterns of |x| (ties to the even pattern), the sign bit added after:
    independent of the oracle's frexp."""
    sign = 0x8000 if x < 0 else 0
    a = abs(x)
    approx = int(np.array([float(a)], np.float32).view(np.uint32)[0] >> 16)
    best = None
    for b in range(max(approx - 2, 0), approx + 3):
        v = Fraction(float(np.array([b << 16], np.uint32).view(np.float32)[0]))
        key = (abs(v - a), b & 1)
        if best is None or key < best[0]:
            best = (key, b)
    return sign | best[1]


def test_single_rounding_against_exact_rationals():
    rng = np.random.default_rng(2201)
    codes = rng.integers(0, 256, 3000).astype(np.uint8)
    codes = codes[(codes & 0x7F) != 0x7F]
    scales = (rng.random(codes.shape[0]) * 2 + 1e-3).astype(np.float32)
    got = dq.bf16_round(dq.e4m3_value(codes) * scales.astype(np.float64))
    for c, s, g in zip(codes, scales, got):
        exact = Fraction(float(dq.e4m3_value(np.array([c]))[0])) * Fraction(float(s))
        want = (0x8000 if c & 0x80 else 0) if exact == 0 else _nearest_bf16_exact(exact)  # signed zeros
        assert g == want, (c, s)


def test_block_scales_follow_the_128_blocks():
    s = np.arange(6, dtype=np.float32).reshape(2, 3) + 1
    full = dq.block_scales(s, 256, 300)
    assert full.shape == (256, 300)
    assert full[0, 0] == 1 and full[127, 127] == 1 and full[128, 0] == 4 and full[0, 128] == 2
    assert full[255, 299] == 6


# ---------------------------------------------------------------- GPU

DEV = torch.device("cuda:0")


@pytest.mark.gpu
@pytest.mark.parametrize("n_heads", [128, 64])
def test_kernel_is_bit_exact_at_the_size_of_wkv_b(n_heads):
    import sparse_latent_attention_absorb_b200 as pkg
    f = wl.generate_fp8_wkv_b(n_heads, seed=2201 + n_heads)
    got = pkg.mla_dequant_fp8_blocks(f["codes"].to(DEV), f["scale"].to(DEV))
    torch.cuda.synchronize()
    want = dq.dequant(f["codes"].numpy(), f["scale"].numpy())
    assert np.array_equal(got.view(torch.int16).cpu().numpy().view(np.uint16), want)


@pytest.mark.gpu
def test_kernel_on_the_hand_derived_and_ragged_cases():
    import sparse_latent_attention_absorb_b200 as pkg
    # one 128 x 128 block per hand case, side by side; then a ragged width
    codes = np.concatenate([np.full((128, 128), c, np.uint8) for c, _, _ in HAND], axis=1)
    scale = np.array([[_scale_value(b) for _, b, _ in HAND]], np.float32)
    got = pkg.mla_dequant_fp8_blocks(torch.from_numpy(codes).to(DEV), torch.from_numpy(scale).to(DEV))
    torch.cuda.synchronize()
    g = got.view(torch.int16).cpu().numpy().view(np.uint16)
    for i, (_, _, want) in enumerate(HAND):
        assert np.all(g[:, 128 * i:128 * (i + 1)] == want)
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 256, (200, 208)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3C
    scale = (rng.random((2, 2)) + 0.1).astype(np.float32)
    got = pkg.mla_dequant_fp8_blocks(torch.from_numpy(codes).to(DEV), torch.from_numpy(scale).to(DEV))
    torch.cuda.synchronize()
    assert np.array_equal(got.view(torch.int16).cpu().numpy().view(np.uint16), dq.dequant(codes, scale))


@pytest.mark.gpu
def test_decode_with_the_dequantised_fp8_weight():
    import oracle
    import sparse_latent_attention_absorb_b200 as pkg
    d = wl.generate("small_b4_ctx600-2k_recent128_top400")
    f = wl.generate_fp8_wkv_b(seed=2299)
    w_bits = dq.dequant(f["codes"].numpy(), f["scale"].numpy())
    w_ref = torch.from_numpy(w_bits.view(np.int16)).view(torch.bfloat16)
    layer = pkg.Fp8Wkvb(f["codes"].to(DEV), f["scale"].to(DEV))
    w = layer.weight()
    assert layer.weight() is w  # built once, then kept
    g = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    out = pkg.mla_sparse_decode(g["q_nope"], g["q_pe"], g["kv_cache"], g["pe_cache"], g["end_pos"], g["topk_idx"], w,
                                g["scale"])
    torch.cuda.synchronize()
    ref = oracle.mla_sparse_decode(d["q_nope"], d["q_pe"], d["kv_cache"], d["pe_cache"], d["end_pos"], d["topk_idx"],
                                   w_ref, d["scale"])
    got = out.double().cpu().numpy()
    assert np.max(np.abs(got - ref.out)) <= 1e-2 * np.max(np.abs(ref.out)) + 1e-3
