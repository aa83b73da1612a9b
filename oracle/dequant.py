"""Oracle of the fp8 block dequantisation of wkv_b (plain numpy).

TEST INFRASTRUCTURE ONLY: imported by the tests, never by the CUDA package.

Page "Query-key similarity" (decode excerpt, model.py 591-592): when wkv_b is
stored in fp8 with a scale, the decode first builds
``self.dequant_wkv_b = weight_dequant(self.wkv_b.weight, self.wkv_b.scale)``
once and uses that weight in place of wkv_b from then on.  The pages do not
print weight_dequant's format; the reading taken here is DeepSeek-V3's block
format: the weight holds OCP FP8 E4M3 codes, the scale one float32 per block of
128 x 128 weights (scale[i, j] for rows [128 i, 128 i + 128) and columns
[128 j, 128 j + 128)), and the dequantised weight, held in bf16 like the rest
of the model, is

    w[r, c] = bf16( value(code[r, c]) * scale[r // 128, c // 128] )

with the product taken exactly and rounded once, to nearest (ties to even).
"""
from __future__ import annotations

import numpy as np

BLOCK = 128


def e4m3_value(codes) -> np.ndarray:
    """float64 values of OCP FP8 E4M3 codes (uint8): sign bit, 4 exponent bits
    (bias 7), 3 mantissa bits; exponent field 0 is subnormal (2^-6 * m/8);
    0x7F and 0xFF are NaN; there is no infinity."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    sub = np.ldexp(m / 8.0, -6)
    v = sign * np.where(e == 0, sub, normal)
    return np.where((c & 0x7F) == 0x7F, np.nan, v)


def bf16_round(x) -> np.ndarray:
    """bf16 bit patterns (uint16) nearest to the float64 values x, ties to
    even (finite inputs within the bf16 normal range, or zero)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                       # x = m * 2^e, 0.5 <= |m| < 1
    q = np.rint(np.ldexp(m, 8))              # 8 significant bits (bf16: 1 + 7), ties to even
    r = np.ldexp(q, e - 8)                   # exactly representable in bf16, hence in float32
    return (r.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def block_scales(scale, rows: int, cols: int) -> np.ndarray:
    """The per-element scale: scale[r // 128, c // 128] as an [rows, cols] array."""
    s = np.asarray(scale, dtype=np.float32).astype(np.float64)
    return np.repeat(np.repeat(s, BLOCK, axis=0), BLOCK, axis=1)[:rows, :cols]


def dequant(codes, scale) -> np.ndarray:
    """The dequantised weight as bf16 bit patterns (uint16), shape of codes."""
    c = np.asarray(codes, dtype=np.uint8)
    rows, cols = c.shape
    return bf16_round(e4m3_value(c) * block_scales(scale, rows, cols))
