// Validation of the top-k index rows (atlas page "Query-key similarity",
// decode excerpt, the index mask of model.py 601-602): the mask is a -inf row
// with 0 scattered at every selected position, so a position listed twice is
// still selected once.  The attention kernel gathers each listed position, so
// it requires the valid entries of a row to be distinct; this kernel finds the
// rows that break that and reports MLA_ERR_BAD_INDEX through the caller's
// status word.  Entries outside [0, min(end_pos, S_max)) are padding, as in
// the decode, and are not checked.
#pragma once

#include <cstdint>

#include "mla_sparse_decode.h"

namespace mla {

constexpr int kCheckThreads = 512;
// Bitmap words in shared memory: one pass covers 32 x this many positions
// (1,048,576); longer rows take several passes over their index row.
constexpr int kCheckMaxWords = 32768;

__host__ __device__ constexpr int check_bitmap_words(int S_max) {
  return (S_max + 31) / 32 < kCheckMaxWords ? (S_max + 31) / 32 : kCheckMaxWords;
}

// One CTA per row b: a bitmap over the row's valid positions; an entry whose
// bit is already set is a repeat.  d_dup (optional) receives 1 for a row with
// a repeat and 0 otherwise.
__global__ void __launch_bounds__(kCheckThreads)
check_indices_kernel(const int32_t* __restrict__ end_pos, const int32_t* __restrict__ topk_idx, int K, int S_max,
                     int* d_status, int* d_dup) {
  extern __shared__ uint32_t bitmap[];
  const int b = blockIdx.x;
  int ep = end_pos[b];
  ep = ep < 0 ? 0 : (ep > S_max ? S_max : ep);
  const int32_t* row = topk_idx + (size_t)b * K;
  const int pass_bits = check_bitmap_words(S_max) * 32;
  bool dup = false;
  for (int base = 0; base < ep; base += pass_bits) {
    const int span = min(ep - base, pass_bits);
    for (int i = threadIdx.x; i < (span + 31) / 32; i += blockDim.x) bitmap[i] = 0u;
    __syncthreads();
    for (int k = threadIdx.x; k < K; k += blockDim.x) {
      const int t = __ldg(row + k);
      if (t >= base && t < base + span) {
        const int off = t - base;
        const uint32_t bit = 1u << (off & 31);
        if (atomicOr(&bitmap[off >> 5], bit) & bit) dup = true;
      }
    }
    __syncthreads();
  }
  const int any = __syncthreads_or(dup ? 1 : 0);
  if (threadIdx.x == 0) {
    if (any && d_status) atomicCAS(d_status, 0, MLA_ERR_BAD_INDEX);
    if (d_dup) d_dup[b] = any ? 1 : 0;
  }
}

}  // namespace mla
