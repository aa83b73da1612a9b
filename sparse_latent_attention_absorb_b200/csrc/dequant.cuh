// fp8 block dequantisation of wkv_b (atlas page "Query-key similarity",
// decode excerpt, model.py 591-592: when wkv_b is stored in fp8 with a scale,
// the decode builds weight_dequant(wkv_b.weight, wkv_b.scale) once and uses
// it in place of wkv_b).  Block format (the pages do not print it; DeepSeek-V3's
// reading): E4M3 codes with one float32 scale per 128 x 128 block, the result
// in bf16:
//   w[r, c] = bf16( e4m3(code[r, c]) * scale[r / 128, c / 128] )
// with the product exact and rounded once, to nearest even.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cstdint>

namespace mla {

constexpr int kDequantBlock = 128;
constexpr int kDequantThreads = 256;

// The exact product p (an e4m3 value times a float32: at most 28 significant
// bits, exact in double) rounded once to bf16: truncate to float32 and set the
// last bit when that dropped anything (round to odd keeps the information a
// second rounding needs: 24 bits >= 8 + 2), then round to nearest even.
__device__ __forceinline__ __nv_bfloat16 round_once_to_bf16(double p) {
  float f = __double2float_rz(p);
  if ((double)f != p) f = __uint_as_float(__float_as_uint(f) | 1u);
  return __float2bfloat16_rn(f);
}

// Sixteen consecutive codes of one row per thread (16-byte load, two 16-byte
// stores); cols is a multiple of 16, so a vector never crosses a row or a
// 128-column block.
__global__ void __launch_bounds__(kDequantThreads)
dequant_fp8_blocks_kernel(const uint8_t* __restrict__ w8, const float* __restrict__ scale,
                          __nv_bfloat16* __restrict__ out, int rows, int cols) {
  const long long n_vec = (long long)rows * (cols / 16);
  const int scale_cols = (cols + kDequantBlock - 1) / kDequantBlock;
  for (long long v = blockIdx.x * (long long)blockDim.x + threadIdx.x; v < n_vec;
       v += (long long)gridDim.x * blockDim.x) {
    const long long e0 = v * 16;
    const int r = (int)(e0 / cols), c = (int)(e0 % cols);
    const double s = (double)__ldg(scale + (size_t)(r / kDequantBlock) * scale_cols + c / kDequantBlock);
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(w8 + e0));
    const uint32_t words[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t packed[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // two codes -> two halves (every E4M3 value is exact in fp16)
        const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(
            static_cast<__nv_fp8x2_storage_t>((words[q] >> (16 * h)) & 0xffffu), __NV_E4M3);
        __half2 h2;
        h2 = *reinterpret_cast<const __half2*>(&hr);
        const float2 f = __half22float2(h2);
        const __nv_bfloat16 lo = round_once_to_bf16((double)f.x * s);
        const __nv_bfloat16 hi = round_once_to_bf16((double)f.y * s);
        packed[2 * q + h] = (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(out + e0);
    dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
  }
}

}  // namespace mla
