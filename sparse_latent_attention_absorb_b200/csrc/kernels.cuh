// sm_100a kernels of the sparse MLA decode step (DeepSeek-V3.2-Exp,
// model.py 590-606 as shown on the atlas pages "Query-key similarity",
// "Softmax" and "Apply value weights").
//
//   absorb_kernel            q_lat = q_nope . W_UK per head        (tcgen05)
//   sparse_attend_kernel     gathered scores, online softmax, mix  (tcgen05,
//                            2-CTA cluster, DSMEM score exchange)
//   combine_value_up_kernel  log-sum-exp merge of the key splits,
//                            then O~ . W_UV^T per head            (tcgen05)
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace mla {

constexpr int kH = MLA_HEADS;         // 128 heads
constexpr int kDn = MLA_D_NOPE;       // 128
constexpr int kDr = MLA_D_ROPE;       // 64
constexpr int kDl = MLA_D_LATENT;     // 512
constexpr int kDv = MLA_D_V;          // 128
constexpr int kHeadRows = kDn + kDv;  // rows of one head in wkv_b

// Dynamic shared memory is only guaranteed 16-byte alignment; 128B-swizzle
// atoms need 1024.  Every kernel requests kSmemAlignPad extra bytes and
// rounds its base up.
constexpr int kSmemAlignPad = 1024;
__device__ __forceinline__ uint8_t* align_smem_1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

// =============================================================================
// absorb_kernel: q_lat[b,h,c] = sum_d q_nope[b,h,d] * W_UK[h,d,c]
//
// Swap-AB GEMM per (head h, 128-column chunk of c, tile of up to 128 rows b):
//   D[c, b] = sum_d W_UK[h, d, c] * q_nope[b, h, d]
// M = 128 (c), N = batch tile (multiple of 16), K = 128 (d).
// A = W_UK[h][:, chunk] is M-major in memory (c contiguous): two TMA boxes of
// 64 c x 128 d, 128B-swizzled.  B = q_nope[:, h, :] is K-major: two 3-D TMA
// boxes of 64 d x N rows.  The accumulator lives in TMEM (lanes = c).
// =============================================================================
constexpr int kAbsorbNMax = 128;
constexpr int kAbsorbSmemA = 2 * 64 * 128 * 2;                      // 32 KB
constexpr int kAbsorbSmemB = 2 * kAbsorbNMax * 128;                  // 32 KB max
constexpr int kAbsorbSmemBytes = kAbsorbSmemA + kAbsorbSmemB + 256 + kSmemAlignPad;  // + barriers

__global__ void __launch_bounds__(128, 1)
absorb_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_q,
              __nv_bfloat16* __restrict__ q_lat, int B, int n_tile, int* d_status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = blockIdx.x;  // 128-wide chunk of the latent dimension
  const int h = blockIdx.y;
  const int b0 = blockIdx.z * kAbsorbNMax;

  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + kAbsorbSmemA;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kAbsorbSmemA + kAbsorbSmemB);
  const uint32_t bar_load = smem_u32(&bars[0]);
  const uint32_t bar_mma = smem_u32(&bars[1]);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&bars[2]);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&bars[3]);
  const AbortState ab{abort_flag, d_status};

  const uint32_t tmem_cols = n_tile <= 32 ? 32u : (n_tile <= 64 ? 64u : 128u);
  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(bar_load, 1);
    mbar_init(bar_mma, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (tid == 0) {
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_q);
    mbar_arrive_expect_tx(bar_load, kAbsorbSmemA + 2 * n_tile * 128);
    const int wrow = h * kHeadRows;  // W_UK rows of head h
    tma_load_2d(sA, &tm_w, bar_load, chunk * 128, wrow);
    tma_load_2d(sA + 64 * 128 * 2, &tm_w, bar_load, chunk * 128 + 64, wrow);
    tma_load_3d(sB, &tm_q, bar_load, 0, h, b0);
    tma_load_3d(sB + n_tile * 128, &tm_q, bar_load, 64, h, b0);

    wait(bar_load, 0, ab);
    tc_fence_after();
    const uint32_t idesc = idesc_bf16_f32(128, n_tile, /*a MN*/ true, /*b MN*/ false);
    for (int k = 0; k < kDn / 16; ++k) {
      // A: 16 d-rows per step (two 8-row groups 1024 B apart); the two
      // 64-wide c blocks are 16 KB apart.
      const uint64_t a = smem_desc_sw128(sA + k * 16 * 128, 64 * 128 * 2, 1024);
      // B: 32 bytes of d per step inside the 128-byte row; the second
      // 64-wide d block follows the first.
      const uint64_t b = smem_desc_sw128(sB + (k >> 2) * n_tile * 128 + (k & 3) * 32, 16, 1024);
      mma_ss(tmem, a, b, idesc, k > 0 ? 1u : 0u);
    }
    mma_commit(bar_mma);
  }
  __syncwarp();

  // Epilogue: lane (32*warp + lane) holds column c of the chunk, one TMEM
  // column per batch row.
  wait(bar_mma, 0, ab);
  tc_fence_after();
  const int c = chunk * 128 + warp * 32 + lane;
  for (int n0 = 0; n0 < n_tile; n0 += 16) {
    uint32_t v[16];
    tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + n0, v);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int b = b0 + n0 + j;
      if (b < B) q_lat[((size_t)b * kH + h) * kDl + c] = __float2bfloat16_rn(__uint_as_float(v[j]));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, tmem_cols);
}

// =============================================================================
// sparse_attend_kernel
//
// One 2-CTA cluster per (batch row b, key split s).  CTA rank r owns latent
// columns [256r, 256r+256) and rotary columns [32r, 32r+32):
//   * it gathers, for every selected position t of the split, kv[b,t,its 256]
//     and pe[b,t,its 32] into shared memory (cp.async, 128B-swizzled rows);
//   * QK: S_r[h,t] = q_lat[h, its 256] . kv[t, its 256] + q_pe[h, its 32] .
//     pe[t, its 32]  -- a split-K half of the 576-wide score, M = 128 heads;
//   * the two halves are exchanged through distributed shared memory, so both
//     CTAs hold the full score S = S_0 + S_1 (bitwise identical in both);
//   * online softmax with a lazily updated running maximum (O is rescaled
//     only when the maximum grows by more than 2^8); P (bf16) goes to TMEM;
//   * PV: O_r[h, its 256] += P[h,t] . kv[t, its 256]  (A = P from TMEM,
//     B = the same gathered rows read M/N-major).
// The split's normalised O and its log-sum-exp go to o_part / lse_part.
//
// Warp roles (288 threads): warps 0-3 softmax (thread i <-> TMEM lane i =
// head i), warp 4 TMEM allocation + MMA issue, warps 5-8 gather.
// =============================================================================
constexpr int kNt = 32;                            // positions per tile
constexpr int kStages = 5;                         // gathered tile ring
constexpr int kLag = kStages - 2;                  // cp.async groups in flight before a tile is published
constexpr int kKB = 5;                             // 128-byte K blocks per row: 4 latent + 1 rotary (half used)
constexpr int kQBytes = kKB * kH * 128;            // 80 KB
constexpr int kStageBytes = kKB * kNt * 128;       // 20 KB
constexpr int kXBytes = (kNt / 4) * kH * 16;       // 16 KB: one exchanged score tile (f32)
constexpr int kOffQ = 0;
constexpr int kOffStage = kOffQ + kQBytes;
constexpr int kOffX = kOffStage + kStages * kStageBytes;
constexpr int kOffBar = kOffX + 2 * kXBytes;
constexpr int kAttendSmemBytes = kOffBar + 256 + kSmemAlignPad;
constexpr int kAttendThreads = 288;
// TMEM columns
constexpr uint32_t kColS = 0;     // two score buffers of kNt columns
constexpr uint32_t kColP = 64;    // two P buffers of kNt/2 columns (bf16 pairs)
constexpr uint32_t kColO = 256;   // 256 columns of O
constexpr float kRescaleThreshold = 8.0f;  // log2 units

static_assert(kOffStage % 1024 == 0 && kStageBytes % 1024 == 0 && kOffX % 1024 == 0, "swizzle atoms");
static_assert(kAttendSmemBytes <= 232448, "shared memory");
static_assert(kLag >= 1, "pipeline");

struct AttendBars {
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];
  uint64_t s_empty[2];
  uint64_t p_full[2];
  uint64_t o_done;
  uint64_t x_full[2];
  uint64_t x_free[2];
  uint32_t tmem_addr;
  int abort_flag;
};
static_assert(sizeof(AttendBars) <= 256, "barrier block");

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kAttendThreads, 1)
sparse_attend_kernel(const __nv_bfloat16* __restrict__ q_lat, const __nv_bfloat16* __restrict__ q_pe,
                     const __nv_bfloat16* __restrict__ kv_cache, const __nv_bfloat16* __restrict__ pe_cache,
                     const int32_t* __restrict__ end_pos, const int32_t* __restrict__ topk_idx, float scale,
                     float* __restrict__ o_part, float* __restrict__ lse_part, int K, int S_max, int n_split,
                     int span, int* d_status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int unit = blockIdx.x >> 1;
  const int b = unit / n_split;
  const int split = unit % n_split;
  const int k_begin = split * span;
  const int k_end = min(K, k_begin + span);
  const int n_tiles = k_end > k_begin ? (k_end - k_begin + kNt - 1) / kNt : 0;
  int ep = end_pos[b];
  ep = ep < 0 ? 0 : (ep > S_max ? S_max : ep);

  const uint32_t sQ = smem_u32(smem + kOffQ);
  const uint32_t sStage = smem_u32(smem + kOffStage);
  const uint32_t sX = smem_u32(smem + kOffX);
  AttendBars* bars = reinterpret_cast<AttendBars*>(smem + kOffBar);
  const AbortState ab{&bars->abort_flag, d_status};

  if (tid == 0) {
    bars->abort_flag = 0;
    mbar_init(smem_u32(&bars->q_full), 128);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_u32(&bars->kv_full[i]), 128);
      mbar_init(smem_u32(&bars->kv_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars->s_full[i]), 1);
      mbar_init(smem_u32(&bars->s_empty[i]), 128);
      mbar_init(smem_u32(&bars->p_full[i]), 128);
      mbar_init(smem_u32(&bars->x_full[i]), 128);
      mbar_init(smem_u32(&bars->x_free[i]), 128);
    }
    mbar_init(smem_u32(&bars->o_done), 1);
    fence_mbarrier_init_cluster();
  }
  if (warp == 4) {
    tmem_alloc(smem_u32(&bars->tmem_addr), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = bars->tmem_addr;

  if (warp >= 5) {
    // ------------------------------------------------------------ gather
    const int ptid = tid - 160;  // 0..127
    const int pw = warp - 5;     // 0..3, 8 positions of each tile
    // Q half: q_lat[b, h, 256r + 8q .. +8] and q_pe[b, h, 32r + 8q .. +8]
    for (int i = ptid; i < kH * 32; i += 128) {
      const int hh = i >> 5, q = i & 31;
      const uint32_t dst = sQ + (q >> 3) * (kH * 128) + sw128_offset(hh, q & 7);
      cp_async_16(dst, q_lat + ((size_t)b * kH + hh) * kDl + rank * 256 + q * 8, 16);
    }
    for (int i = ptid; i < kH * 4; i += 128) {
      const int hh = i >> 2, q = i & 3;
      const uint32_t dst = sQ + 4 * (kH * 128) + sw128_offset(hh, q);
      cp_async_16(dst, q_pe + ((size_t)b * kH + hh) * kDr + rank * 32 + q * 8, 16);
    }
    cp_async_commit();

    const __nv_bfloat16* kv_row0 = kv_cache + (size_t)b * S_max * kDl + rank * 256;
    const __nv_bfloat16* pe_row0 = pe_cache + (size_t)b * S_max * kDr + rank * 32;
    for (int j = 0; j < n_tiles; ++j) {
      const int st = j % kStages;
      if (j >= kStages) wait(smem_u32(&bars->kv_empty[st]), ((j / kStages) - 1) & 1, ab);
      const uint32_t stage = sStage + st * kStageBytes;
      // lanes 0..7 fetch the indices of this warp's 8 positions
      int idx = -1;
      if (lane < 8) {
        const int k = k_begin + j * kNt + pw * 8 + lane;
        if (k < k_end) idx = topk_idx[(size_t)b * K + k];
      }
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int n = pw * 8 + t;  // row of the tile
        const int pos = __shfl_sync(0xffffffffu, idx, t);
        const bool valid = pos >= 0 && pos < ep;
        const size_t p = valid ? (size_t)pos : 0;
        // latent: lane l copies 16 bytes = 8 columns [8l, 8l+8) of the half
        {
          const uint32_t dst = stage + (lane >> 3) * (kNt * 128) + sw128_offset(n, lane & 7);
          cp_async_16(dst, kv_row0 + p * kDl + lane * 8, valid ? 16u : 0u);
        }
        if (lane < 4) {
          const uint32_t dst = stage + 4 * (kNt * 128) + sw128_offset(n, lane);
          cp_async_16(dst, pe_row0 + p * kDr + lane * 8, valid ? 16u : 0u);
        }
      }
      cp_async_commit();
      if (j >= kLag) {
        cp_async_wait_group<kLag>();
        fence_proxy_async_smem();
        const int jt = j - kLag;
        if (jt == 0) mbar_arrive(smem_u32(&bars->q_full));
        mbar_arrive(smem_u32(&bars->kv_full[jt % kStages]));
      }
    }
    cp_async_wait_all();
    fence_proxy_async_smem();
    for (int jt = n_tiles - kLag < 0 ? 0 : n_tiles - kLag; jt < n_tiles; ++jt) {
      if (jt == 0) mbar_arrive(smem_u32(&bars->q_full));
      mbar_arrive(smem_u32(&bars->kv_full[jt % kStages]));
    }
    if (n_tiles == 0) mbar_arrive(smem_u32(&bars->q_full));
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0 && n_tiles > 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(128, kNt, false, false);
      const uint32_t idesc_pv = idesc_bf16_f32(128, 256, false, true);
      wait(smem_u32(&bars->q_full), 0, ab);
      auto issue_pv = [&](int t) {
        wait(smem_u32(&bars->p_full[t & 1]), (t >> 1) & 1, ab);
        tc_fence_after();
        const uint32_t stage = sStage + (t % kStages) * kStageBytes;
#pragma unroll
        for (int k = 0; k < kNt / 16; ++k) {
          // B = gathered latent rows read N-major: 16 positions per step,
          // the four 64-column blocks kNt*128 bytes apart.
          const uint64_t bdesc = smem_desc_sw128(stage + k * 16 * 128, kNt * 128, 1024);
          mma_ts(tmem + kColO, tmem + kColP + (t & 1) * (kNt / 2) + k * 8, bdesc, idesc_pv,
                 (t > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(smem_u32(&bars->kv_empty[t % kStages]));
        mma_commit(smem_u32(&bars->o_done));
      };
      for (int j = 0; j < n_tiles; ++j) {
        const int st = j % kStages;
        wait(smem_u32(&bars->kv_full[st]), (j / kStages) & 1, ab);
        if (j >= 2) wait(smem_u32(&bars->s_empty[j & 1]), ((j >> 1) - 1) & 1, ab);
        tc_fence_after();
        const uint32_t stage = sStage + st * kStageBytes;
#pragma unroll
        for (int k = 0; k < 18; ++k) {
          const int kb = k < 16 ? (k >> 2) : 4;
          const int within = (k < 16 ? (k & 3) : (k - 16)) * 32;
          const uint64_t adesc = smem_desc_sw128(sQ + kb * (kH * 128) + within, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(stage + kb * (kNt * 128) + within, 16, 1024);
          mma_ss(tmem + kColS + (j & 1) * kNt, adesc, bdesc, idesc_qk, k > 0 ? 1u : 0u);
        }
        mma_commit(smem_u32(&bars->s_full[j & 1]));
        if (j >= 1) issue_pv(j - 1);
      }
      issue_pv(n_tiles - 1);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int i = tid;  // head
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const float c2 = scale * 1.4426950408889634f;  // scores to log2 units
    float m_used = -INFINITY, l_sum = 0.f;
    uint32_t x_peer[2], xfull_peer[2], xfree_peer[2];
    for (int u = 0; u < 2; ++u) {
      x_peer[u] = cluster_map(sX + u * kXBytes, peer);
      xfull_peer[u] = cluster_map(smem_u32(&bars->x_full[u]), peer);
      xfree_peer[u] = cluster_map(smem_u32(&bars->x_free[u]), peer);
    }
    for (int j = 0; j < n_tiles; ++j) {
      const int u = j & 1;
      // validity of the tile's positions (same in every softmax warp)
      int pos = -1;
      {
        const int k = k_begin + j * kNt + lane;
        if (k < k_end) pos = topk_idx[(size_t)b * K + k];
      }
      const uint32_t vmask = __ballot_sync(0xffffffffu, pos >= 0 && pos < ep);

      wait(smem_u32(&bars->s_full[u]), (j >> 1) & 1, ab);
      tc_fence_after();
      uint32_t sv[32];
      tmem_ld32(tmem + lane_base + kColS + u * kNt, sv);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(smem_u32(&bars->s_empty[u]));

      // exchange the split-K halves of the score tile with the peer CTA
      if (j >= 2) wait_cluster(smem_u32(&bars->x_free[u]), ((j >> 1) - 1) & 1, ab);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint32_t a = x_peer[u] + (uint32_t)((q * kH + i) * 16);
        asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(sv[4 * q]),
                     "r"(sv[4 * q + 1]), "r"(sv[4 * q + 2]), "r"(sv[4 * q + 3])
                     : "memory");
      }
      mbar_arrive_remote(xfull_peer[u]);
      wait_cluster(smem_u32(&bars->x_full[u]), (j >> 1) & 1, ab);
      float s[32];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 o = *reinterpret_cast<const float4*>(smem + kOffX + u * kXBytes + (q * kH + i) * 16);
        s[4 * q + 0] = __uint_as_float(sv[4 * q + 0]) + o.x;
        s[4 * q + 1] = __uint_as_float(sv[4 * q + 1]) + o.y;
        s[4 * q + 2] = __uint_as_float(sv[4 * q + 2]) + o.z;
        s[4 * q + 3] = __uint_as_float(sv[4 * q + 3]) + o.w;
      }
      mbar_arrive_remote(xfree_peer[u]);

      // online softmax in log2 units
      float mx = -INFINITY;
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        s[t] = ((vmask >> t) & 1u) ? s[t] * c2 : -INFINITY;
        mx = fmaxf(mx, s[t]);
      }
      // The running maximum of a row moves only when the tile's maximum
      // exceeds it by more than 2^8 (so p <= 256 otherwise).  The TMEM
      // accesses are warp-collective, so the whole warp rescales when any of
      // its rows must; rows that keep their maximum use alpha = 1.
      const bool grow = mx > m_used + kRescaleThreshold;
      const float alpha = grow ? ((m_used == -INFINITY) ? 0.f : ex2_approx(m_used - mx)) : 1.f;
      if (__any_sync(0xffffffffu, grow) && j > 0) {
        // PV(j-1) must have finished before O is rescaled in place
        wait(smem_u32(&bars->o_done), (j - 1) & 1, ab);
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t ov[32];
          tmem_ld32(tmem + lane_base + kColO + cc * 32, ov);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; ++t) ov[t] = __float_as_uint(__uint_as_float(ov[t]) * alpha);
          tmem_st32(tmem + lane_base + kColO + cc * 32, ov);
        }
        tmem_wait_st();
      }
      l_sum *= alpha;
      if (grow) m_used = mx;
      uint32_t pk[16];
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        const bool v0 = (vmask >> (2 * t)) & 1u, v1 = (vmask >> (2 * t + 1)) & 1u;
        const float p0 = v0 ? ex2_approx(s[2 * t] - m_used) : 0.f;
        const float p1 = v1 ? ex2_approx(s[2 * t + 1] - m_used) : 0.f;
        pk[t] = pack_bf16x2(p0, p1);
        const float2 r = unpack_bf16x2(pk[t]);  // the values the MMA will use
        l_sum += r.x + r.y;
      }
      tmem_st16(tmem + lane_base + kColP + u * (kNt / 2), pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&bars->p_full[u]));
    }

    // epilogue: normalised O half and log-sum-exp of this split
    float* orow = o_part + (((size_t)b * n_split + split) * kH + i) * kDl + rank * 256;
    if (n_tiles > 0) {
      wait(smem_u32(&bars->o_done), (n_tiles - 1) & 1, ab);
      tc_fence_after();
    }
    const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
#pragma unroll 1
    for (int cc = 0; cc < 8; ++cc) {
      uint32_t ov[32];
      if (n_tiles > 0) {
        tmem_ld32(tmem + lane_base + kColO + cc * 32, ov);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int t = 0; t < 32; ++t) ov[t] = 0u;
      }
#pragma unroll
      for (int t = 0; t < 32; t += 4) {
        float4 v = make_float4(__uint_as_float(ov[t]) * inv, __uint_as_float(ov[t + 1]) * inv,
                               __uint_as_float(ov[t + 2]) * inv, __uint_as_float(ov[t + 3]) * inv);
        *reinterpret_cast<float4*>(orow + cc * 32 + t) = v;
      }
    }
    if (rank == 0) {
      lse_part[((size_t)b * n_split + split) * kH + i] =
          l_sum > 0.f ? (m_used + log2f(l_sum)) * 0.6931471805599453f : -INFINITY;
    }
  }

  // teardown: all TMEM traffic done, then release TMEM; keep both CTAs alive
  // until neither can touch the other's shared memory any more.
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 4) tmem_dealloc(tmem, 512);
  cluster_sync();
}

// =============================================================================
// combine_value_up_kernel
//
// Per (head h, tile of up to 64 rows b):
//   coefficients a_s = exp(lse_s - L) with L = log sum_s exp(lse_s);
//   O~[b, :] = sum_s a_s o_part[b, s, h, :], rounded to bf16 into shared memory
//   (K-major B operand, 128B-swizzled);
//   D[e, b] = sum_c W_UV[h, e, c] * O~[b, c]   (M = 128 value dims, K = 512)
//   with W_UV[h] (128 KB) brought in by eight TMA boxes.
// =============================================================================
constexpr int kCombineNMax = 64;
constexpr int kCombineMaxSplits = 128;
constexpr int kCombineSmemA = 8 * 128 * 128;             // 128 KB
constexpr int kCombineSmemB = 8 * kCombineNMax * 128;    // 64 KB
constexpr int kCombineSmemCoef = kCombineNMax * kCombineMaxSplits * 4;  // 32 KB
constexpr int kCombineSmemBytes = kCombineSmemA + kCombineSmemB + kCombineSmemCoef + 256 + kSmemAlignPad;
constexpr int kCombineThreads = 256;
static_assert(kCombineSmemBytes <= 232448, "shared memory");

__global__ void __launch_bounds__(kCombineThreads, 1)
combine_value_up_kernel(const __grid_constant__ CUtensorMap tm_w, const float* __restrict__ o_part,
                        const float* __restrict__ lse_part, __nv_bfloat16* __restrict__ out,
                        float* __restrict__ lse_out, int B, int n_split, int n_tile, int* d_status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x;
  const int b0 = blockIdx.y * kCombineNMax;
  const int rows = min(kCombineNMax, B - b0);

  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + kCombineSmemA;
  float* coef = reinterpret_cast<float*>(smem + kCombineSmemA + kCombineSmemB);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kCombineSmemA + kCombineSmemB + kCombineSmemCoef);
  const uint32_t bar_w = smem_u32(&bars[0]);
  const uint32_t bar_mma = smem_u32(&bars[1]);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&bars[2]);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(&bars[3]);
  const AbortState ab{abort_flag, d_status};
  const uint32_t tmem_cols = n_tile <= 32 ? 32u : 64u;

  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(bar_w, 1);
    mbar_init(bar_mma, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (tid == 0) {
    tma_prefetch_desc(&tm_w);
    mbar_arrive_expect_tx(bar_w, kCombineSmemA);
    const int wrow = h * kHeadRows + kDn;  // W_UV rows of head h
    for (int kb = 0; kb < 8; ++kb) tma_load_2d(sA + kb * 128 * 128, &tm_w, bar_w, kb * 64, wrow);
  }

  // split weights, one row per thread
  if (tid < rows) {
    const int b = b0 + tid;
    float mx = -INFINITY;
    for (int s = 0; s < n_split; ++s) mx = fmaxf(mx, lse_part[((size_t)b * n_split + s) * kH + h]);
    float total = 0.f;
    for (int s = 0; s < n_split; ++s) {
      const float l = lse_part[((size_t)b * n_split + s) * kH + h];
      const float w = (mx == -INFINITY) ? 0.f : __expf(l - mx);
      coef[tid * kCombineMaxSplits + s] = w;
      total += w;
    }
    const float inv = total > 0.f ? 1.f / total : 0.f;
    for (int s = 0; s < n_split; ++s) coef[tid * kCombineMaxSplits + s] *= inv;
    if (lse_out) lse_out[(size_t)b * kH + h] = total > 0.f ? mx + __logf(total) : -INFINITY;
  }
  __syncthreads();

  // merged O~ rows -> bf16 K-major operand (row n = batch row, 512 columns)
  for (int it = tid; it < n_tile * 64; it += kCombineThreads) {
    const int n = it >> 6, q = it & 63;  // q: 8-column chunk of the 512
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (n < rows) {
      const int b = b0 + n;
      for (int s = 0; s < n_split; ++s) {
        const float a = coef[n * kCombineMaxSplits + s];
        const float4* src = reinterpret_cast<const float4*>(o_part + (((size_t)b * n_split + s) * kH + h) * kDl + q * 8);
        const float4 x0 = src[0], x1 = src[1];
        acc[0] += a * x0.x; acc[1] += a * x0.y; acc[2] += a * x0.z; acc[3] += a * x0.w;
        acc[4] += a * x1.x; acc[5] += a * x1.y; acc[6] += a * x1.z; acc[7] += a * x1.w;
      }
    }
    const uint32_t dst = sB + (q >> 3) * (n_tile * 128) + sw128_offset(n, q & 7);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(pack_bf16x2(acc[0], acc[1])),
                 "r"(pack_bf16x2(acc[2], acc[3])), "r"(pack_bf16x2(acc[4], acc[5])),
                 "r"(pack_bf16x2(acc[6], acc[7]))
                 : "memory");
  }
  fence_proxy_async_smem();
  __syncthreads();

  if (tid == 0) {
    wait(bar_w, 0, ab);
    tc_fence_after();
    const uint32_t idesc = idesc_bf16_f32(128, n_tile, false, false);
    for (int k = 0; k < kDl / 16; ++k) {
      const uint64_t a = smem_desc_sw128(sA + (k >> 2) * (128 * 128) + (k & 3) * 32, 16, 1024);
      const uint64_t bd = smem_desc_sw128(sB + (k >> 2) * (n_tile * 128) + (k & 3) * 32, 16, 1024);
      mma_ss(tmem, a, bd, idesc, k > 0 ? 1u : 0u);
    }
    mma_commit(bar_mma);
  }
  __syncwarp();

  if (warp < 4) {
    wait(bar_mma, 0, ab);
    tc_fence_after();
    const int e = warp * 32 + lane;  // value dimension
    for (int n0 = 0; n0 < n_tile; n0 += 16) {
      uint32_t v[16];
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + n0, v);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int n = n0 + j;
        if (n < rows) out[((size_t)(b0 + n) * kH + h) * kDv + e] = __float2bfloat16_rn(__uint_as_float(v[j]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, tmem_cols);
}

}  // namespace mla
